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

// ---------------------------------------------------------------- keys in registers
//
// reg_select: n <= NT * KPT keys, key_at(u) of thread t being the key of index u * NT + t
// (key 0 past n and for absent candidates), from registers or shared memory; every pass
// is unrolled over u, so a thread's reads are all in flight together.  Same selection
// rule as above.
//   1. range: hi = the largest key, lo = the larger of lo_key (a caller's lower bound on
//      the k-th key, 0 if none) and the smallest valid key;
//   2. one histogram of RSEL_BINS linear bins over [lo, hi] (a monotone fp32 map) and
//      a scan from the top bin find the bin holding the k-th key;
//   3. the keys of that bin are gathered and ranked exactly (a bin of one key value
//      needs no ranking);
//   4. one counting pass and one emit pass, with exclusive prefixes of the per-(u, warp)
//      counts, output the selection in index order.
// Passes run over the ceil(n / NT) index steps that hold keys, with modest unrolling
// (fully unrolled passes made the code large enough to stall on instruction fetch).  Returns the number selected
// and the threshold key T (the k-th key; T == 0 when every valid key is selected), or -1
// (CTA-uniform) when the boundary bin holds more than RSEL_CAP distinct-valued keys, in
// which case nothing has been emitted and the caller falls back to the passes above.

constexpr int RSEL_BINS = 4096;
constexpr int RSEL_CAP = 1024;           // boundary-bin keys ranked in shared memory
constexpr int RSEL_RANK_MAX = 256;       // up to this many: rank by direct comparison

template <int NT, int KPT>
struct RegSelectShared {
    unsigned hist[RSEL_BINS];
    unsigned bkey[RSEL_CAP];
    unsigned cnt_gt[KPT][NT / 32];       // per (u, warp) counts, then exclusive prefixes
    unsigned cnt_eq[KPT][NT / 32];
    unsigned wmax[NT / 32], wmin[NT / 32], wsum[NT / 32];
    SelectShared<NT> sel;                // radix scratch for a large boundary bin
    unsigned lo, hi, bstar, above, n_gather, bmin, bmax, T, need_eq, total_gt, total_eq;
    int status;
};

template <int NT, int KPT, class KeyAt, class EmitFn>
__device__ __forceinline__ int reg_select(const KeyAt& key_at, int n, int k, unsigned lo_key,
                                          RegSelectShared<NT, KPT>& sh, unsigned& T_out,
                                          const EmitFn& emit) {
    static_assert(NT % 32 == 0 && RSEL_BINS % 32 == 0, "whole warps");
    constexpr int NW = NT / 32;
    constexpr int BPT = (RSEL_BINS + NT - 1) / NT;       // bins per thread in the scan
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int nu = min(KPT, (n + NT - 1) / NT);          // index steps holding keys

    // ---- 1. range (and cleared histogram)
    unsigned mx = 0u, mn = 0xFFFFFFFFu;
#pragma unroll 4
    for (int u = 0; u < nu; ++u) {
        const unsigned kk = key_at(u);
        if (kk != 0u && kk >= lo_key) {
            mx = max(mx, kk);
            mn = min(mn, kk);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
    }
    if (lane == 0) {
        sh.wmax[warp] = mx;
        sh.wmin[warp] = mn;
    }
    for (int i = tid; i < RSEL_BINS; i += NT) sh.hist[i] = 0u;
    if (tid == 0) {
        sh.n_gather = 0u;
        sh.bmin = 0xFFFFFFFFu;
        sh.bmax = 0u;
        sh.status = 0;
    }
    __syncthreads();
    unsigned hi = 0u, lo = 0xFFFFFFFFu;
    for (int w = 0; w < NW; ++w) {
        hi = max(hi, sh.wmax[w]);
        lo = min(lo, sh.wmin[w]);
    }
    if (hi == 0u) {                                       // nothing valid at or above lo_key
        T_out = 0u;
        __syncthreads();
        return 0;
    }
    // bin = floor((kk - lo) * BINS / (hi - lo + 1)) in fp32: every step (int -> float,
    // the multiply, the truncation) is monotone non-decreasing, which is all the
    // selection needs (a higher bin never holds a smaller key)
    const float bin_scale = static_cast<float>(RSEL_BINS) / (static_cast<float>(hi - lo) + 1.0f);
    const auto bin_of = [&](unsigned kk) {
        return min(static_cast<unsigned>(static_cast<float>(kk - lo) * bin_scale),
                   static_cast<unsigned>(RSEL_BINS - 1));
    };

    // ---- 2. histogram, then the bin holding the k-th key (scan from the top bin)
#pragma unroll 4
    for (int u = 0; u < nu; ++u) {
        const unsigned kk = key_at(u);
        if (kk != 0u && kk >= lo) atomicAdd(&sh.hist[bin_of(kk)], 1u);
    }
    __syncthreads();
    unsigned seg = 0;                                    // bins RSEL_BINS-1-BPT*tid downwards
    for (int i = 0; i < BPT; ++i) {
        const int b = RSEL_BINS - 1 - BPT * tid - i;
        if (b >= 0) seg += sh.hist[b];
    }
    unsigned incl = seg;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) sh.wsum[warp] = incl;
    __syncthreads();
    unsigned before = 0, total = 0;
    for (int w = 0; w < NW; ++w) {
        if (w < warp) before += sh.wsum[w];
        total += sh.wsum[w];
    }
    const unsigned kk_sel = static_cast<unsigned>(k);
    if (total <= kk_sel) {                                // every key >= lo is selected
        if (tid == 0) {
            sh.T = lo - 1u;                               // keys > T == keys >= lo
            sh.need_eq = 0u;
        }
    } else {
        const unsigned excl = before + incl - seg;
        if (excl < kk_sel && kk_sel <= excl + seg) {
            unsigned cum = excl;
            for (int i = 0; i < BPT; ++i) {
                const int b = RSEL_BINS - 1 - BPT * tid - i;
                if (b < 0) break;
                if (cum + sh.hist[b] >= kk_sel) {
                    sh.bstar = static_cast<unsigned>(b);
                    sh.above = cum;
                    break;
                }
                cum += sh.hist[b];
            }
        }
        __syncthreads();
        // ---- 3. the boundary bin's keys
        const unsigned bstar = sh.bstar;
#pragma unroll 4
        for (int u = 0; u < nu; ++u) {
            const unsigned kk = key_at(u);
            if (kk != 0u && kk >= lo && bin_of(kk) == bstar) {
                const unsigned j = atomicAdd(&sh.n_gather, 1u);
                if (j < RSEL_CAP) sh.bkey[j] = kk;
                atomicMin(&sh.bmin, kk);
                atomicMax(&sh.bmax, kk);
            }
        }
        __syncthreads();
        const unsigned m = sh.n_gather;
        const unsigned need = kk_sel - sh.above;          // 1 <= need <= m
        if (sh.bmin == sh.bmax) {                         // one value: it is the k-th key
            if (tid == 0) {
                sh.T = sh.bmin;
                sh.need_eq = need;
            }
        } else if (m <= RSEL_RANK_MAX) {
            for (unsigned j = tid; j < m; j += NT) {
                const unsigned v = sh.bkey[j];
                unsigned gt = 0, ge = 0;
                for (unsigned i = 0; i < m; ++i) {
                    gt += sh.bkey[i] > v;
                    ge += sh.bkey[i] >= v;
                }
                if (gt < need && need <= ge) {            // every such thread writes the same
                    sh.T = v;
                    sh.need_eq = need - gt;
                }
            }
        } else if (m <= RSEL_CAP) {
            unsigned T;
            int need_eq;
            const auto bk = [&](int j) { return sh.bkey[j]; };
            radix_threshold<NT>(bk, static_cast<int>(m), static_cast<int>(need), sh.sel, T, need_eq);
            if (tid == 0) {
                sh.T = T;
                sh.need_eq = static_cast<unsigned>(need_eq);
            }
        } else if (tid == 0) {
            sh.status = -1;
        }
    }
    __syncthreads();
    if (sh.status != 0) {
        __syncthreads();
        return -1;
    }
    const unsigned T = sh.T;
    const unsigned need_eq = sh.need_eq;
    T_out = T;

    // ---- 4. per-(u, warp) counts, exclusive prefixes in index order, ordered emit
#pragma unroll 4
    for (int u = 0; u < nu; ++u) {
        const unsigned gt = __ballot_sync(0xFFFFFFFFu, key_at(u) > T);
        const unsigned eq = __ballot_sync(0xFFFFFFFFu, key_at(u) == T && T != 0u);
        if (lane == 0) {
            sh.cnt_gt[u][warp] = __popc(gt);
            sh.cnt_eq[u][warp] = __popc(eq);
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int E = nu * NW;
        const int PER = (E + 31) / 32;                    // entries per lane, in order
        unsigned sg = 0, se = 0;
        for (int i = 0; i < PER; ++i) {
            const int e = lane * PER + i;
            if (e < E) {
                sg += (&sh.cnt_gt[0][0])[e];
                se += (&sh.cnt_eq[0][0])[e];
            }
        }
        unsigned ig = sg, ie = se;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned yg = __shfl_up_sync(0xFFFFFFFFu, ig, off);
            const unsigned ye = __shfl_up_sync(0xFFFFFFFFu, ie, off);
            if (lane >= off) {
                ig += yg;
                ie += ye;
            }
        }
        unsigned rg = ig - sg, re = ie - se;
        for (int i = 0; i < PER; ++i) {
            const int e = lane * PER + i;
            if (e < E) {
                const unsigned cg = (&sh.cnt_gt[0][0])[e], ce = (&sh.cnt_eq[0][0])[e];
                (&sh.cnt_gt[0][0])[e] = rg;
                (&sh.cnt_eq[0][0])[e] = re;
                rg += cg;
                re += ce;
            }
        }
        if (lane == 31) {
            sh.total_gt = ig;
            sh.total_eq = ie;
        }
    }
    __syncthreads();
#pragma unroll 4
    for (int u = 0; u < nu; ++u) {
        const bool is_gt = key_at(u) > T;
        const bool is_eq = key_at(u) == T && T != 0u;
        const unsigned gt = __ballot_sync(0xFFFFFFFFu, is_gt);
        const unsigned eq = __ballot_sync(0xFFFFFFFFu, is_eq);
        const unsigned eq_rank = sh.cnt_eq[u][warp] + __popc(eq & lt_mask);
        if (is_gt || (is_eq && eq_rank < need_eq)) {
            const unsigned slot = sh.cnt_gt[u][warp] + __popc(gt & lt_mask) + min(eq_rank, need_eq);
            emit(u * NT + tid, static_cast<int>(slot));
        }
    }
    const int n_sel = static_cast<int>(sh.total_gt + min(sh.total_eq, need_eq));
    __syncthreads();                                      // scratch is reused by the caller
    return n_sel;
}


// ---------------------------------------------------------------- staging

// Copies n floats from global src to shared dst (16-byte aligned), each thread keeping
// STAGE_BATCH loads in flight before it stores them (a load-store loop waits one memory
// latency per iteration).
constexpr int STAGE_BATCH = 8;

template <int NT>
__device__ __forceinline__ void stage_floats(float* dst, const float* __restrict__ src, int n) {
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
        const int n4 = n >> 2;
        const float4* s4 = reinterpret_cast<const float4*>(src);
        float4* d4 = reinterpret_cast<float4*>(dst);
        for (int base = threadIdx.x; base < n4; base += NT * STAGE_BATCH) {
            float4 v[STAGE_BATCH];
#pragma unroll
            for (int b = 0; b < STAGE_BATCH; ++b) {
                const int i = base + b * NT;
                v[b] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int b = 0; b < STAGE_BATCH; ++b) {
                const int i = base + b * NT;
                if (i < n4) d4[i] = v[b];
            }
        }
        for (int i = 4 * n4 + static_cast<int>(threadIdx.x); i < n; i += NT) dst[i] = __ldg(src + i);
    } else {
        for (int base = threadIdx.x; base < n; base += NT * STAGE_BATCH) {
            float v[STAGE_BATCH];
#pragma unroll
            for (int b = 0; b < STAGE_BATCH; ++b) {
                const int i = base + b * NT;
                v[b] = i < n ? __ldg(src + i) : 0.0f;
            }
#pragma unroll
            for (int b = 0; b < STAGE_BATCH; ++b) {
                const int i = base + b * NT;
                if (i < n) dst[i] = v[b];
            }
        }
    }
}

// ---------------------------------------------------------------- keys in shared memory,
// with a lower bound: the fast path of the chunk selects
//
// fast_select: the same selection rule, for n keys readable as key_of(i) and a caller's
// lower bound lo_key on the k-th key (0 if none).  Built for throughput with few warps:
//   A. survivors (valid keys >= lo_key) counted per lane over each warp's contiguous
//      segment, FS_ILP loads in flight, no votes;
//   B. survivors compacted (key, index) in index order, FS_ILP 32-key chunks per step
//      (independent ballots, one running offset per step);
//   C. the k-th survivor: one histogram of FS_BINS linear bins over [lo, hi] of the
//      survivors, the boundary bin's keys ranked exactly (a bin of one value needs none);
//   D. the selected survivors emitted in index order (ballots over the short list).
// Returns the number selected and the threshold key T (T == 0: every valid key), or -1
// (CTA-uniform, nothing emitted) when more than FS_CAP keys survive or the boundary bin
// holds more than FS_RANK distinct keys: the caller then runs the general passes.

constexpr int FS_ILP = 8;
constexpr int FS_BINS = 2048;
constexpr int FS_CAP = 2048;
constexpr int FS_RANK = 256;

template <int NT>
struct FastSelectShared {
    unsigned hist[FS_BINS];
    unsigned key[FS_CAP];                 // survivors in index order
    uint16_t idx[FS_CAP];
    unsigned bkey[FS_RANK];
    unsigned wtot[NT / 32], wtot2[NT / 32];
    unsigned bstar, above, n_gather, bmin, bmax, T, need_eq;
};

template <int NT, class KeyFn, class EmitFn>
__device__ __forceinline__ int fast_select(const KeyFn& key_of, int n, int k, unsigned lo_key,
                                           FastSelectShared<NT>& sh, unsigned& T_out, const EmitFn& emit) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const unsigned lt_mask = (1u << lane) - 1u;
    const unsigned floor_key = lo_key == 0u ? 0u : lo_key - 1u;   // survivors: key > floor_key
    // warp w owns [seg_lo, seg_hi), a multiple of 32 * FS_ILP long
    const int seg = ((n + NW - 1) / NW + 32 * FS_ILP - 1) / (32 * FS_ILP) * (32 * FS_ILP);
    const int seg_lo = min(warp * seg, n), seg_hi = min(seg_lo + seg, n);

    // ---- A. count survivors (and their range) per lane
    unsigned cnt = 0, mx = 0u, mn = 0xFFFFFFFFu;
    for (int base = seg_lo; base < seg_hi; base += 32 * FS_ILP) {
        unsigned kk[FS_ILP];
#pragma unroll
        for (int u = 0; u < FS_ILP; ++u) {
            const int i = base + 32 * u + lane;
            kk[u] = i < seg_hi ? key_of(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < FS_ILP; ++u) {
            const bool s = kk[u] > floor_key;
            cnt += s;
            if (s) {
                mx = max(mx, kk[u]);
                mn = min(mn, kk[u]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, off);
        mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
    }
    if (lane == 0) sh.wtot[warp] = cnt;
    __syncthreads();
    unsigned before = 0, total = 0;
    for (int w = 0; w < NW; ++w) {
        const unsigned c = sh.wtot[w];
        if (w < warp) before += c;
        total += c;
    }
    __syncthreads();                                     // wtot is reused below
    if (total > static_cast<unsigned>(FS_CAP)) return -1;   // uniform: nothing emitted
    const int m = static_cast<int>(total);

    // ---- B. ordered compaction of the survivors
    {
        unsigned out = before;
        for (int base = seg_lo; base < seg_hi; base += 32 * FS_ILP) {
            unsigned kk[FS_ILP], bal[FS_ILP];
#pragma unroll
            for (int u = 0; u < FS_ILP; ++u) {
                const int i = base + 32 * u + lane;
                kk[u] = i < seg_hi ? key_of(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < FS_ILP; ++u) bal[u] = __ballot_sync(0xFFFFFFFFu, kk[u] > floor_key);
#pragma unroll
            for (int u = 0; u < FS_ILP; ++u) {
                if (kk[u] > floor_key) {
                    const unsigned slot = out + __popc(bal[u] & lt_mask);
                    sh.key[slot] = kk[u];
                    sh.idx[slot] = static_cast<uint16_t>(base + 32 * u + lane);
                }
                out += __popc(bal[u]);
            }
        }
    }
    // survivor range (every warp's lanes agree on mx / mn after the shuffles)
    if (lane == 0) {
        sh.wtot[warp] = mx;
        sh.wtot2[warp] = mn;
    }
    for (int i = tid; i < FS_BINS; i += NT) sh.hist[i] = 0u;
    if (tid == 0) {
        sh.n_gather = 0u;
        sh.bmin = 0xFFFFFFFFu;
        sh.bmax = 0u;
    }
    __syncthreads();
    unsigned hi = 0u, lo = 0xFFFFFFFFu;
    for (int w = 0; w < NW; ++w) {
        hi = max(hi, sh.wtot[w]);
        lo = min(lo, sh.wtot2[w]);
    }
    unsigned T, need_eq;
    const unsigned kk_sel = static_cast<unsigned>(k);
    if (m <= k) {                                        // every survivor is selected
        T = m == 0 ? 0xFFFFFFFFu : lo - 1u;
        need_eq = 0u;
        __syncthreads();                                 // the range reads of wtot are done
    } else {
        // ---- C. histogram of the survivors, the boundary bin, exact rank inside it
        const float bin_scale = static_cast<float>(FS_BINS) / (static_cast<float>(hi - lo) + 1.0f);
        const auto bin_of = [&](unsigned key) {
            return min(static_cast<unsigned>(static_cast<float>(key - lo) * bin_scale),
                       static_cast<unsigned>(FS_BINS - 1));
        };
        for (int j = tid; j < m; j += NT) atomicAdd(&sh.hist[bin_of(sh.key[j])], 1u);
        __syncthreads();
        constexpr int BPT = (FS_BINS + NT - 1) / NT;
        unsigned segsum = 0;
        for (int i = 0; i < BPT; ++i) {
            const int b = FS_BINS - 1 - BPT * tid - i;
            if (b >= 0) segsum += sh.hist[b];
        }
        unsigned incl = segsum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) sh.wtot[warp] = incl;
        __syncthreads();
        unsigned wbefore = 0;
        for (int w = 0; w < warp; ++w) wbefore += sh.wtot[w];
        const unsigned excl = wbefore + incl - segsum;
        if (excl < kk_sel && kk_sel <= excl + segsum) {
            unsigned cum = excl;
            for (int i = 0; i < BPT; ++i) {
                const int b = FS_BINS - 1 - BPT * tid - i;
                if (b < 0) break;
                if (cum + sh.hist[b] >= kk_sel) {
                    sh.bstar = static_cast<unsigned>(b);
                    sh.above = cum;
                    break;
                }
                cum += sh.hist[b];
            }
        }
        __syncthreads();
        const unsigned bstar = sh.bstar;
        for (int j = tid; j < m; j += NT) {
            const unsigned key = sh.key[j];
            if (bin_of(key) == bstar) {
                const unsigned g = atomicAdd(&sh.n_gather, 1u);
                if (g < FS_RANK) sh.bkey[g] = key;
                atomicMin(&sh.bmin, key);
                atomicMax(&sh.bmax, key);
            }
        }
        __syncthreads();
        const unsigned mb = sh.n_gather;
        const unsigned need = kk_sel - sh.above;
        if (sh.bmin == sh.bmax) {
            T = sh.bmin;
            need_eq = need;
        } else if (mb <= static_cast<unsigned>(FS_RANK)) {
            for (unsigned j = tid; j < mb; j += NT) {
                const unsigned v = sh.bkey[j];
                unsigned gt = 0, ge = 0;
                for (unsigned i = 0; i < mb; ++i) {
                    gt += sh.bkey[i] > v;
                    ge += sh.bkey[i] >= v;
                }
                if (gt < need && need <= ge) {
                    sh.T = v;
                    sh.need_eq = need - gt;
                }
            }
            __syncthreads();
            T = sh.T;
            need_eq = sh.need_eq;
        } else {
            __syncthreads();
            return -1;
        }
    }
    T_out = T == 0xFFFFFFFFu ? 0u : T;

    // ---- D. emit the selected survivors in index order
    {
        const int s_lo = min(tid * ((m + NT - 1) / NT), m);
        const int s_hi = min(s_lo + (m + NT - 1) / NT, m);   // this thread's survivors
        // per-thread counts of selected (gt) and tied (eq) survivors, then block prefixes
        unsigned cg = 0, ce = 0;
        for (int j = s_lo; j < s_hi; ++j) {
            const unsigned key = sh.key[j];
            cg += key > T && T != 0xFFFFFFFFu;
            ce += key == T;
        }
        unsigned ig = cg, ie = ce;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned yg = __shfl_up_sync(0xFFFFFFFFu, ig, off);
            const unsigned ye = __shfl_up_sync(0xFFFFFFFFu, ie, off);
            if (lane >= off) {
                ig += yg;
                ie += ye;
            }
        }
        if (lane == 31) {
            sh.wtot[warp] = ig;
            sh.wtot2[warp] = ie;
        }
        __syncthreads();
        unsigned bg = 0, be = 0, tg = 0, te = 0;
        for (int w = 0; w < NW; ++w) {
            if (w < warp) {
                bg += sh.wtot[w];
                be += sh.wtot2[w];
            }
            tg += sh.wtot[w];
            te += sh.wtot2[w];
        }
        unsigned og = bg + ig - cg, oe = be + ie - ce;   // before this thread's range
        for (int j = s_lo; j < s_hi; ++j) {
            const unsigned key = sh.key[j];
            const bool gt = key > T && T != 0xFFFFFFFFu;
            const bool eq = key == T;
            if (gt || (eq && oe < need_eq)) emit(static_cast<int>(sh.idx[j]), static_cast<int>(og + min(oe, need_eq)));
            og += gt;
            oe += eq;
        }
        const int n_sel = T == 0xFFFFFFFFu ? 0 : static_cast<int>(tg + min(te, need_eq));
        __syncthreads();
        return n_sel;
    }
}

}  // namespace csa2
