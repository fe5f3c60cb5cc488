// CTA-wide exact Top-k selection (device side), shared by the fused indexer scan, the
// candidate merge, the stage-level Top-K and the HSI pool.
//
// Selection rule (the CSA2 pages give no tie rule): keep the k largest keys; among equal
// keys the lower index wins.  Keys are the monotone 32-bit images of fp32 scores
// (score_key); key 0 marks an absent candidate and is never selected.
//
//   radix_threshold: MSB-first radix select, 4 passes of 8 bits.  Histogram updates are
//     aggregated per warp (__match_any_sync) so keys sharing a digit cost one shared
//     atomic per warp.  Result: threshold T and need_eq such that the selection is every
//     key > T plus the first need_eq keys == T in index order (T == 0: every valid key).
//   stable_emit: each warp owns a contiguous segment of the index range, walks it 32
//     keys at a time (coalesced, bank-conflict free) and ranks selected keys with
//     ballots, so outputs come out in index order.
//   global_select: for keys in global memory.  One pass builds a 12-bit histogram of the
//     top key bits; the keys at or above the boundary bin (usually a few hundred) are
//     compacted, in index order, into shared memory, where the exact select finishes.
//     If the boundary bin is too large for shared memory it falls back to running the
//     two routines above on the global keys.
// Loads are batched UNROLL deep per lane so that each warp keeps several in flight.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int SEL_UNROLL = 4;

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
    static_assert(NT >= 64 && NT % 32 == 0, "select needs whole warps");
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    unsigned prefix = 0u, mask = 0u;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += NT) sh.hist[i] = 0u;
        __syncthreads();
        // warp-uniform trip count: lanes past n take part with key 0
        for (int base = tid - lane; base < n; base += NT * SEL_UNROLL) {
            unsigned key[SEL_UNROLL];
#pragma unroll
            for (int u = 0; u < SEL_UNROLL; ++u) {
                const int i = base + u * NT + lane;
                key[u] = i < n ? key_of(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < SEL_UNROLL; ++u) {
                const bool match = key[u] != 0u && (key[u] & mask) == prefix;
                const unsigned active = __ballot_sync(0xFFFFFFFFu, match);
                if (match) {
                    const unsigned d = (key[u] >> shift) & 255u;
                    const unsigned peers = __match_any_sync(active, d);
                    if (lane == __ffs(peers) - 1) atomicAdd(&sh.hist[d], static_cast<unsigned>(__popc(peers)));
                }
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
    constexpr int STEP = 32 * SEL_UNROLL;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int seg = ((n + NW - 1) / NW + STEP - 1) / STEP * STEP;
    const int lo = min(warp * seg, n);
    const int hi = min(lo + seg, n);
    const unsigned lt_mask = (1u << lane) - 1u;

    int gt = 0, eq = 0;
    for (int base = lo; base < hi; base += STEP) {
        unsigned key[SEL_UNROLL];
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            const int i = base + 32 * u + lane;
            key[u] = i < hi ? key_of(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            gt += __popc(__ballot_sync(0xFFFFFFFFu, key[u] > T));
            eq += __popc(__ballot_sync(0xFFFFFFFFu, T != 0u && key[u] == T));
        }
    }
    if (lane == 0) {
        sh.warp_a[warp] = gt;
        sh.warp_b[warp] = eq;
    }
    __syncthreads();
    int eq_before = 0, sel_before = 0, total = 0, my_eq_before = 0;
    for (int w = 0; w < NW; ++w) {
        const int e = sh.warp_b[w];
        const int take = max(0, min(need_eq - eq_before, e));
        const int sel = sh.warp_a[w] + take;
        if (w < warp) {
            sel_before += sel;
            my_eq_before += e;
        }
        total += sel;
        eq_before += e;
    }
    int eq_budget = max(0, min(need_eq - my_eq_before, eq));   // ties this warp may take
    int out = sel_before;
    for (int base = lo; base < hi; base += STEP) {
        unsigned key[SEL_UNROLL];
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            const int i = base + 32 * u + lane;
            key[u] = i < hi ? key_of(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            const int i = base + 32 * u + lane;
            const bool is_eq = T != 0u && key[u] == T;
            const unsigned eqm = __ballot_sync(0xFFFFFFFFu, is_eq);
            const bool take_eq = is_eq && __popc(eqm & lt_mask) < eq_budget;
            const bool sel = key[u] > T || take_eq;
            const unsigned selm = __ballot_sync(0xFFFFFFFFu, sel);
            if (sel) emit(i, out + __popc(selm & lt_mask));
            out += __popc(selm);
            eq_budget = max(0, eq_budget - __popc(eqm));
        }
    }
    __syncthreads();          // shared scratch is reused by the caller
    return total;
}

// ---------------------------------------------------------------- keys in global memory

constexpr int GSEL_CAP = 8192;           // boundary candidates kept in shared memory

template <int NT>
struct alignas(128) GlobalSelectShared {
    unsigned hist[4096];                 // 12-bit histogram of the first pass
    unsigned key[GSEL_CAP];              // compacted candidates, in index order
    int idx[GSEL_CAP];
    SelectShared<NT> sel;
    unsigned boundary, above, total;
};

// Selects the Top-k of key_of(0 .. n-1) and calls emit(i, slot) in increasing i.
template <int NT, class KeyFn, class EmitFn>
__device__ __forceinline__ int global_select(const KeyFn& key_of, int n, int k,
                                             GlobalSelectShared<NT>& sh, const EmitFn& emit) {
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    for (int i = tid; i < 4096; i += NT) sh.hist[i] = 0u;
    __syncthreads();
    for (int base = tid - lane; base < n; base += NT * SEL_UNROLL) {
        unsigned key[SEL_UNROLL];
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            const int i = base + u * NT + lane;
            key[u] = i < n ? key_of(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < SEL_UNROLL; ++u) {
            const bool valid = key[u] != 0u;
            const unsigned active = __ballot_sync(0xFFFFFFFFu, valid);
            if (valid) {
                const unsigned d = key[u] >> 20;
                const unsigned peers = __match_any_sync(active, d);
                if (lane == __ffs(peers) - 1) atomicAdd(&sh.hist[d], static_cast<unsigned>(__popc(peers)));
            }
        }
    }
    __syncthreads();
    if (tid < 32) {
        // lane l owns bins 4095-128l .. 3968-128l (descending)
        unsigned part = 0;
        for (int i = 0; i < 128; ++i) part += sh.hist[4095 - 128 * lane - i];
        unsigned incl = part;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        const unsigned excl = incl - part;
        if (lane == 31) sh.total = incl;
        const unsigned kk = static_cast<unsigned>(k);
        if (excl < kk && kk <= incl) {
            unsigned cum = excl;
            for (int i = 0; i < 128; ++i) {
                const unsigned bin = 4095 - 128 * lane - i;
                if (cum + sh.hist[bin] >= kk) {
                    sh.boundary = bin;
                    sh.above = cum + sh.hist[bin];          // candidates at or above it
                    break;
                }
                cum += sh.hist[bin];
            }
        }
    }
    __syncthreads();
    if (sh.total <= static_cast<unsigned>(k))             // every valid key is selected
        return stable_emit<NT>(key_of, n, 0u, 0, sh.sel, emit);
    const unsigned bnd = sh.boundary;
    const int n_cand = static_cast<int>(sh.above);
    if (n_cand > GSEL_CAP) {                               // fall back to global passes
        unsigned T;
        int need_eq;
        radix_threshold<NT>(key_of, n, k, sh.sel, T, need_eq);
        return stable_emit<NT>(key_of, n, T, need_eq, sh.sel, emit);
    }
    // keys in bins >= bnd, compacted in index order
    const unsigned floor_key = bnd == 0u ? 0u : (bnd << 20) - 1u;
    stable_emit<NT>(key_of, n, floor_key, 0, sh.sel, [&](int i, int slot) {
        sh.key[slot] = key_of(i);
        sh.idx[slot] = i;
    });
    const auto ckey = [&](int j) { return sh.key[j]; };
    unsigned T;
    int need_eq;
    radix_threshold<NT>(ckey, n_cand, k, sh.sel, T, need_eq);
    return stable_emit<NT>(ckey, n_cand, T, need_eq, sh.sel,
                           [&](int j, int slot) { emit(sh.idx[j], slot); });
}

}  // namespace csa2
