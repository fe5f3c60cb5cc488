// CTA-wide exact Top-k selection (device side), shared by the fused indexer scan, the
// candidate merge, the stage-level Top-K and the HSI pool.
//
// Selection rule (the CSA2 pages give no tie rule): keep the k largest keys; among equal
// keys the lower index wins.  Keys are the monotone 32-bit images of fp32 scores
// (score_key); key 0 marks an absent candidate and is never selected.
//
//   radix_threshold: MSB-first radix select, 4 passes of 8 bits.  Histogram updates are
//     aggregated per warp (__match_any_sync) so that keys sharing a digit - most of them
//     in the first pass - cost one shared-memory atomic per warp instead of one each.
//     Result: threshold T and need_eq such that the selection is every key > T plus the
//     first need_eq keys == T in index order (T == 0 means "every valid key").
//   stable_emit: each warp owns a contiguous segment of the index range, walks it 32
//     keys at a time (coalesced, bank-conflict free) and ranks selected keys with
//     ballots, so outputs come out in index order.
#pragma once

#include "common.cuh"

namespace csa2 {

template <int NT>
struct SelectShared {
    unsigned hist[256];
    int warp_a[NT / 32];
    int warp_b[NT / 32];
    unsigned digit, above, total;
};

// All NT threads must call with the same n, k.  key_of(i) for 0 <= i < n.
template <int NT, class KeyFn>
__device__ __forceinline__ void radix_threshold(const KeyFn& key_of, int n, int k,
                                                SelectShared<NT>& sh, unsigned& T, int& need_eq) {
    static_assert(NT >= 256 && NT % 32 == 0, "select needs >= 256 threads");
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    unsigned prefix = 0u, mask = 0u;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += NT) sh.hist[i] = 0u;
        __syncthreads();
        // warp-uniform trip count: lanes past n take part with match = false
        for (int base = tid - lane; base < n; base += NT) {
            const int i = base + lane;
            const unsigned key = i < n ? key_of(i) : 0u;
            const bool match = key != 0u && (key & mask) == prefix;
            const unsigned active = __ballot_sync(0xFFFFFFFFu, match);
            if (match) {
                const unsigned d = (key >> shift) & 255u;
                const unsigned peers = __match_any_sync(active, d);
                if (lane == __ffs(peers) - 1) atomicAdd(&sh.hist[d], static_cast<unsigned>(__popc(peers)));
            }
        }
        __syncthreads();
        if (tid < 32) {
            unsigned part = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) part += sh.hist[255 - 8 * lane - i];
            unsigned incl = part;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += y;
            }
            const unsigned excl = incl - part;
            if (lane == 31) sh.total = incl;
            const unsigned rem = static_cast<unsigned>(remaining);
            if (excl < rem && rem <= incl) {
                unsigned cum = excl;
                for (int i = 0; i < 8; ++i) {
                    const unsigned bin = 255 - 8 * lane - i;
                    if (cum + sh.hist[bin] >= rem) {
                        sh.digit = bin;
                        sh.above = cum;
                        break;
                    }
                    cum += sh.hist[bin];
                }
            }
        }
        __syncthreads();
        if (pass == 0 && sh.total <= static_cast<unsigned>(k)) {
            T = 0u;
            need_eq = 0;
            return;
        }
        remaining -= static_cast<int>(sh.above);
        prefix |= sh.digit << shift;
        mask |= 0xFFu << shift;
    }
    T = prefix;
    need_eq = remaining;
}

// Emits the selected indices in increasing order: emit(i, slot), slot = 0, 1, ...
// Returns the number selected (same value in every thread).
template <int NT, class KeyFn, class EmitFn>
__device__ __forceinline__ int stable_emit(const KeyFn& key_of, int n, unsigned T, int need_eq,
                                           SelectShared<NT>& sh, const EmitFn& emit) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int seg = ((n + NW - 1) / NW + 31) / 32 * 32;
    const int lo = min(warp * seg, n);
    const int hi = min(lo + seg, n);
    const unsigned lt_mask = (1u << lane) - 1u;

    int gt = 0, eq = 0;
    for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const unsigned key = i < hi ? key_of(i) : 0u;
        gt += __popc(__ballot_sync(0xFFFFFFFFu, key > T));
        eq += __popc(__ballot_sync(0xFFFFFFFFu, T != 0u && key == T));
    }
    if (lane == 0) {
        sh.warp_a[warp] = gt;
        sh.warp_b[warp] = eq;
    }
    __syncthreads();
    int eq_before = 0, sel_before = 0, total = 0;
    for (int w = 0; w < NW; ++w) {
        const int e = sh.warp_b[w];
        const int take = max(0, min(need_eq - eq_before, e));
        const int sel = sh.warp_a[w] + take;
        if (w < warp) sel_before += sel;
        total += sel;
        eq_before += e;
    }
    int my_eq_before = 0;
    for (int w = 0; w < warp; ++w) my_eq_before += sh.warp_b[w];
    int eq_budget = max(0, min(need_eq - my_eq_before, eq));   // ties this warp may take
    int out = sel_before;
    for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const unsigned key = i < hi ? key_of(i) : 0u;
        const bool is_eq = T != 0u && key == T;
        const unsigned eqm = __ballot_sync(0xFFFFFFFFu, is_eq);
        const bool take_eq = is_eq && __popc(eqm & lt_mask) < eq_budget;
        const bool sel = key > T || take_eq;
        const unsigned selm = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) emit(i, out + __popc(selm & lt_mask));
        out += __popc(selm);
        eq_budget = max(0, eq_budget - __popc(eqm));
    }
    __syncthreads();          // shared scratch is reused by the caller
    return total;
}

}  // namespace csa2
