// topk.cu -- K1 (gate normaliser + hard top-K per row) and K1b (selection bitmap).
//
// Selection rule (SAS study note 1-2, TopK eq.; arXiv text 3 Preliminaries):
// keep the min(K, C) highest scores among a row's C historical candidates;
// equal scores go to the lower block index; output ascending. The gate
// normaliser is log sum_{i<C} exp s_i (study note 2-1 gate eq.; arXiv text 4,
// normalised gate), and the kept blocks' log-gates are s_i minus it.
//
// Exactness: scores are compared through an order-preserving uint32 key, so the
// K-th largest key is found exactly (a bit search over the keys, MSB first,
// narrowed first by a bound or a histogram of the top bits). The keys above it
// are kept, and the ones equal to it are kept in index order until K are
// chosen. Rows of up to 512 candidates take one warp, longer (decode) rows a
// whole CTA; either way a thread owns the strided candidates thread,
// thread + width, ..., so index order is (slot, thread) order and per-slot
// ballots give the tie ranks and output positions.
#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

// log g of a kept block with score x under gate activation `mode` (arXiv text
// 4, design elements: normalised, independent and raw-logit gates; hard gate
// with a straight-through gradient; study note 3-3, 3-4). lse is the
// normaliser over the C candidates, lse_sel the one over the kept blocks.
__device__ __forceinline__ float gate_logit_of(int mode, float x, float lse, float lse_sel) {
    switch (mode) {
        case SAS_GATE_SOFTMAX: return x - lse;
        case SAS_GATE_SIGMOID: return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
        case SAS_GATE_RAW: return x;
        case SAS_GATE_SOFTMAX_SELECTED: return x - lse_sel;
        default: return 0.f;   // none; hard gate: g = 1 on every kept block
    }
}

// Position of row `row` (query t): q_offset + t, or, with per-sequence cache
// lengths (decode rows, T = 1), the new token of sequence b: lens[b] - 1.
__device__ __forceinline__ int64_t row_position(const Shape& sh, const int32_t* lens, int64_t row, int t) {
    if (lens == nullptr) return (int64_t)sh.q_offset + t;
    const int64_t b = row / ((int64_t)sh.Hkv * sh.T);
    const int64_t n = lens[b];   // clamped to [1, q_offset + 1]: the scores row holds NB blocks
    return (n < 1 ? 1 : (n > (int64_t)sh.q_offset + 1 ? (int64_t)sh.q_offset + 1 : n)) - 1;
}

// One warp per row for rows of at most 32 * SLOTS candidates (several rows per
// CTA). Lane l owns candidates l, l + 32, l + 64, ... (coalesced loads; index
// order is (slot, lane) order, so ties and output positions come from per-slot
// ballots). When K <= 32, the K-th largest of the 32 lane maxima (a warp
// bitonic sort) is a key that at least K candidates reach; the keys at or
// above it (normally a few dozen) are compacted into shared memory, four per
// lane, and a warp bitonic sort of those <= 128 keys gives the K-th largest
// directly. Rows with more than 128 such keys, or K > 32, run a bit search
// over all their keys from the highest bit where the bound and the row
// maximum differ. A row takes only the slots its C candidates
// need (4, 8, 12 or 16 per lane): causal training rows have anywhere from 0
// to NB - 1 candidates, and every per-slot step costs instructions.
constexpr int kWarpCap = 128;                    // compacted keys per warp

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <int SLOTS>
__device__ __forceinline__ void topk_warp_row(const Shape& sh, const float* __restrict__ scores, int64_t row, int C,
                                              uint32_t* __restrict__ s_cand, int32_t* __restrict__ idx_out,
                                              float* __restrict__ gl_out, float* __restrict__ lse_out,
                                              int32_t* __restrict__ nsel_out) {
    constexpr int kCap = kWarpCap;
    const int lane = threadIdx.x & 31;
    const int K = sh.K;
    const int n = C < K ? C : K;
    const float* srow = scores + row * sh.NB;
    const uint32_t lt = (1u << lane) - 1u;

    uint32_t key[SLOTS];
    float mloc = -INFINITY, xs[SLOTS];
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const int i = lane + 32 * k;
        xs[k] = i < C ? srow[i] : -INFINITY;
        key[k] = i < C ? float_key(xs[k]) : 0u;  // below every valid key (float_key(-inf) = 0x007fffff)
        mloc = fmaxf(mloc, xs[k]);
    }
    // gate normaliser: lse = m + log sum exp(s - m)
    const float m = warp_max(mloc);
    float lsum = 0.f;
    if (m != -INFINITY) {
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (lane + 32 * k < C) lsum += exp2f((xs[k] - m) * kLog2e);
    }
    lsum = warp_sum(lsum);
    const float lse = (C > 0 && m != -INFINITY) ? m + logf(lsum) : -INFINITY;

    // the n-th largest key; `need` of its copies are kept
    uint32_t thr = 0;
    if (n > 0 && n == C) {
        // every candidate is kept: the threshold is the smallest key
        uint32_t mn = 0xffffffffu;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (lane + 32 * k < C) mn = min(mn, key[k]);
        thr = __reduce_min_sync(0xffffffffu, mn);
    } else if (n > 0) {
        uint32_t lmax = 0;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) lmax = max(lmax, key[k]);
        const uint32_t hi = __reduce_max_sync(0xffffffffu, lmax);
        bool compact = false, small = false;
        uint32_t lo = 0, rank = (uint32_t)n;   // the threshold is the rank-th largest compacted key
        if (n <= 32) {
            // bitonic sort of the lane maxima, descending across lanes
            uint32_t v = lmax;
#pragma unroll
            for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                for (int stride = size >> 1; stride > 0; stride >>= 1) {
                    const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
                    const bool up = (lane & size) == 0;         // descending runs
                    const bool lower = (lane & stride) == 0;
                    v = (lower == up) ? max(v, o) : min(v, o);
                }
            }
            // the smallest i with #{keys >= v_i} >= n (i = n - 1 always
            // qualifies: v_0 .. v_{n-1} are the maxima of n different lanes,
            // valid keys since n < C); then v_{i-1} > v_i, and the n-th
            // largest key lies in [v_i, v_{i-1})
            int ia = 0, ib = n - 1;
            while (ia < ib) {                                     // warp-uniform
                const int mid = (ia + ib) >> 1;
                const uint32_t vm = __shfl_sync(0xffffffffu, v, mid);
                uint32_t c = 0;
#pragma unroll
                for (int k = 0; k < SLOTS; ++k) c += key[k] >= vm ? 1u : 0u;
                if (warp_sum_u32(c) >= (uint32_t)n) ib = mid; else ia = mid + 1;
            }
            lo = __shfl_sync(0xffffffffu, v, ia);
            const uint32_t upv = __shfl_sync(0xffffffffu, v, ia > 0 ? ia - 1 : 0);
            const bool has_up = ia > 0;
            // the keys at or above v_{i-1} are all kept; the ones in
            // [v_i, v_{i-1}) are compacted, and the threshold is the
            // (n - #above)-th largest of them
            uint32_t ca = 0, cnt = 0;
#pragma unroll
            for (int k = 0; k < SLOTS; ++k) {
                const bool over = has_up && key[k] >= upv;
                ca += over ? 1u : 0u;
                cnt += (key[k] >= lo && !over) ? 1u : 0u;
            }
            rank = (uint32_t)n - warp_sum_u32(ca);
            uint32_t incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
            compact = total <= (uint32_t)kCap;
            small = total <= 32u;
            if (compact) {
                uint32_t at = incl - cnt;
#pragma unroll
                for (int k = 0; k < SLOTS; ++k)
                    if (key[k] >= lo && !(has_up && key[k] >= upv)) s_cand[at++] = key[k];
                const uint32_t fill = small ? 32u : (uint32_t)kCap;
                for (uint32_t e = total + lane; e < fill; e += 32) s_cand[e] = 0u;
                __syncwarp();
            }
        }
        if (compact && small) {
            // at most 32 keys, one per lane: a 32-wide bitonic sort, descending
            uint32_t w1 = s_cand[lane];
#pragma unroll
            for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                for (int stride = size >> 1; stride > 0; stride >>= 1) {
                    const uint32_t o = __shfl_xor_sync(0xffffffffu, w1, stride);
                    const bool up = (lane & size) == 0;
                    const bool lower = (lane & stride) == 0;
                    w1 = (lower == up) ? max(w1, o) : min(w1, o);
                }
            }
            thr = __shfl_sync(0xffffffffu, w1, (int)rank - 1);
        } else if (compact) {
            // at most 128 keys, four per lane: a 128-wide bitonic sort, descending
            uint32_t v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = s_cand[lane + 32 * e];
#pragma unroll
            for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
                for (int j = k >> 1; j > 0; j >>= 1) {
                    if (j >= 32) {
                        const int js = j >> 5;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            if (e & js) continue;
                            const bool up = ((lane + 32 * e) & k) == 0;
                            const uint32_t a = v[e], b = v[e | js];
                            v[e] = up ? max(a, b) : min(a, b);
                            v[e | js] = up ? min(a, b) : max(a, b);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t o = __shfl_xor_sync(0xffffffffu, v[e], j);
                            const bool up = ((lane + 32 * e) & k) == 0;
                            const bool lower = (lane & j) == 0;
                            v[e] = (lower == up) ? max(v[e], o) : min(v[e], o);
                        }
                    }
                }
            }
            const int pos = (int)rank - 1;
            const int ps = pos >> 5;
            const uint32_t mine = ps == 0 ? v[0] : ps == 1 ? v[1] : ps == 2 ? v[2] : v[3];
            thr = __shfl_sync(0xffffffffu, mine, pos & 31);
        } else {
            // bit search for the largest v with #{keys >= v} >= n, starting
            // below the prefix that lo and hi share (every v in [lo, hi] has it)
            const uint32_t diff = lo ^ hi;
            const int top = diff == 0u ? -1 : 31 - __clz(diff);
            thr = top >= 31 ? 0u : (hi & ~((2u << top) - 1u));
            if (top < 0) thr = hi;
            for (int bit = top; bit >= 0; --bit) {
                const uint32_t cand = thr | (1u << bit);
                uint32_t c = 0;
#pragma unroll
                for (int k = 0; k < SLOTS; ++k) c += key[k] >= cand ? 1u : 0u;
                if (warp_sum_u32(c) >= (uint32_t)n) thr = cand;
            }
        }
    }
    // keep every key above thr and the first `need` copies of thr in index
    // order (all of them when that is every copy: no tie ranks needed)
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const bool valid = n > 0 && lane + 32 * k < C;
        gt += (valid && key[k] > thr) ? 1u : 0u;
        eq += (valid && key[k] == thr) ? 1u : 0u;
    }
    const uint32_t need = (uint32_t)n - warp_sum_u32(gt);
    const bool all_eq = warp_sum_u32(eq) == need;
    int32_t* io = idx_out + row * K;
    float* go = gl_out + row * K;
    uint32_t take_bits = 0;
    if (all_eq) {
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (n > 0 && lane + 32 * k < C && key[k] >= thr) take_bits |= 1u << k;
    } else {
        uint32_t eq_run = 0;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) {
            const int i = lane + 32 * k;
            const bool valid = n > 0 && i < C;
            const uint32_t eqb = __ballot_sync(0xffffffffu, valid && key[k] == thr);
            if (valid && (key[k] > thr || (key[k] == thr && eq_run + __popc(eqb & lt) < need))) take_bits |= 1u << k;
            eq_run += __popc(eqb);
        }
    }
    float lse_sel = 0.f;
    if (sh.gate == SAS_GATE_SOFTMAX_SELECTED) {      // normaliser over the kept blocks
        float mk = -INFINITY;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if ((take_bits >> k) & 1u) mk = fmaxf(mk, xs[k]);
        mk = warp_max(mk);
        float sk = 0.f;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if ((take_bits >> k) & 1u) sk += expf(xs[k] - mk);
        lse_sel = mk + logf(warp_sum(sk));
    }
    uint32_t pos_run = 0;
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const bool take = (take_bits >> k) & 1u;
        const uint32_t tb = __ballot_sync(0xffffffffu, take);
        if (take) {
            const uint32_t pos = pos_run + __popc(tb & lt);
            io[pos] = lane + 32 * k;
            go[pos] = gate_logit_of(sh.gate, xs[k], lse, lse_sel);
        }
        pos_run += __popc(tb);
    }
    for (int jj = n + lane; jj < K; jj += 32) { io[jj] = -1; go[jj] = 0.f; }
    if (lane == 0) { lse_out[row] = lse; nsel_out[row] = n; }
}

template <int SLOTS>
__global__ void __launch_bounds__(256)
block_topk_warp_kernel(Shape sh, const float* __restrict__ scores, const int32_t* __restrict__ lens,
                       int32_t* __restrict__ idx_out, float* __restrict__ gl_out, float* __restrict__ lse_out,
                       int32_t* __restrict__ nsel_out) {
    __shared__ uint32_t s_cand[8][kWarpCap];
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * 8 + warp;
    if (row >= sh.rows()) return;                // warp-uniform
    // 32-bit index arithmetic where it fits (training rows: a few per cent of the call)
    const bool r32 = sh.rows() <= (int64_t)UINT32_MAX;
    const int t = r32 ? (int)((uint32_t)row % (uint32_t)sh.T) : (int)(row % sh.T);
    const int C = (lens == nullptr && r32) ? (int)(((uint32_t)sh.q_offset + (uint32_t)t) / (uint32_t)sh.bs)
                                           : (int)(row_position(sh, lens, row, t) / sh.bs);
    if (SLOTS > 4 && C <= 128)
        topk_warp_row<4>(sh, scores, row, C, s_cand[warp], idx_out, gl_out, lse_out, nsel_out);
    else if (SLOTS > 8 && C <= 256)
        topk_warp_row<8>(sh, scores, row, C, s_cand[warp], idx_out, gl_out, lse_out, nsel_out);
    else if (SLOTS > 12 && C <= 384)
        topk_warp_row<12>(sh, scores, row, C, s_cand[warp], idx_out, gl_out, lse_out, nsel_out);
    else
        topk_warp_row<SLOTS>(sh, scores, row, C, s_cand[warp], idx_out, gl_out, lse_out, nsel_out);
}

template <int SLOTS>
cudaError_t run_topk_warp(const Shape& s, const float* scores, const int32_t* lens, int32_t* idx, float* gl,
                          float* lse, int32_t* nsel, cudaStream_t st) {
    const int64_t grid = (s.rows() + 7) / 8;
    KernelTimer kt("block_topk", st);
    cudaError_t e = launch_pdl(block_topk_warp_kernel<SLOTS>, dim3((unsigned)grid), dim3(256), 0, st, s, scores, lens,
                               idx, gl, lse, nsel);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

// One CTA of NT threads per row, for long rows (decode rows of up to NT * 8
// candidates). Thread t owns candidates t, t + NT, ... (coalesced loads; index
// order is (slot, thread) order). The K-th largest key: a 2048-bin histogram of
// the keys' top 11 bits picks the bin that holds it; the keys of that bin
// (normally a handful) are compacted into shared memory and one warp finishes
// with a bit search over the 21 bits below. When that bin holds more keys than
// the compaction buffer (long runs of equal scores), the search narrows by
// further histogram passes over 11 and then 10 bits among the keys that match
// so far. Kept keys are then placed in index order by per-slot ballots and one
// cross-warp prefix.
template <int NT, int SLOTS>
__global__ void __launch_bounds__(NT)
block_topk_cta_kernel(Shape sh, const float* __restrict__ scores, const int32_t* __restrict__ lens,
                      int32_t* __restrict__ idx_out, float* __restrict__ gl_out, float* __restrict__ lse_out,
                      int32_t* __restrict__ nsel_out) {
    constexpr int kW = NT / 32;
    constexpr int kBins = 2048;
    constexpr int kCand = 1024;
    __shared__ __align__(16) uint32_t s_hist[kBins];
    __shared__ uint32_t s_cand[kCand];
    __shared__ float s_rm[kW], s_rs[kW];
    __shared__ uint32_t s_cnt[SLOTS][kW];
    __shared__ uint32_t s_misc[8];       // digit, need-in-bin, candidates, thr, need, prefix, mask, overflow
    __shared__ float s_lse;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();
    pdl_wait();
    const int64_t row = blockIdx.x;
    const int t = (int)(row % sh.T);
    const int64_t p = row_position(sh, lens, row, t);
    const int C = (int)(p / sh.bs);
    const int K = sh.K;
    const int n = C < K ? C : K;
    const float* srow = scores + row * sh.NB;
    const uint32_t lt = (1u << lane) - 1u;

    for (int e = tid; e < kBins; e += NT) s_hist[e] = 0u;
    if (tid == 0) s_misc[2] = 0u;
    uint32_t key[SLOTS];
    float xs[SLOTS], mloc = -INFINITY;
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const int i = tid + NT * k;
        xs[k] = i < C ? srow[i] : -INFINITY;
        key[k] = i < C ? float_key(xs[k]) : 0u;
        mloc = fmaxf(mloc, xs[k]);
    }
    // gate normaliser: (max, sum of exp) pairs reduced in one pass
    float msum = mloc, ssum = 0.f;
    if (mloc != -INFINITY) {
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (tid + NT * k < C) ssum += exp2f((xs[k] - mloc) * kLog2e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, msum, o), s2 = __shfl_xor_sync(0xffffffffu, ssum, o);
        const float mm = fmaxf(msum, m2);
        ssum = (msum == -INFINITY ? 0.f : ssum * exp2f((msum - mm) * kLog2e)) +
               (m2 == -INFINITY ? 0.f : s2 * exp2f((m2 - mm) * kLog2e));
        msum = mm;
    }
    if (lane == 0) { s_rm[warp] = msum; s_rs[warp] = ssum; }
    // histogram of the top 11 key bits
#pragma unroll
    for (int k = 0; k < SLOTS; ++k)
        if (tid + NT * k < C) atomicAdd(&s_hist[key[k] >> 21], 1u);
    __syncthreads();
    if (warp == 1) {
        // the warps' (max, sum) pairs, one per lane, reduced by warp 1 while
        // warp 0 scans the histogram; read by the others after the barriers below
        float m = lane < kW ? s_rm[lane] : -INFINITY, sm = lane < kW ? s_rs[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sm, o);
            const float mm = fmaxf(m, m2);
            sm = (m == -INFINITY ? 0.f : sm * exp2f((m - mm) * kLog2e)) +
                 (m2 == -INFINITY ? 0.f : s2 * exp2f((m2 - mm) * kLog2e));
            m = mm;
        }
        if (lane == 0) s_lse = (C > 0 && m != -INFINITY) ? m + logf(sm) : -INFINITY;
    }

    // ---- the n-th largest key: radix passes of 11, 11, 10 bits until its bin is small ----
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)n, thr = 0;
    if (n > 0) {
        int shift = 21;
        for (int pass = 0; pass < 3; ++pass) {
            const int bits = pass < 2 ? 11 : 10;
            if (pass > 0) {
                for (int e = tid; e < kBins; e += NT) s_hist[e] = 0u;
                __syncthreads();
#pragma unroll
                for (int k = 0; k < SLOTS; ++k)
                    if (tid + NT * k < C && (key[k] & pmask) == prefix)
                        atomicAdd(&s_hist[(key[k] >> shift) & ((1u << bits) - 1u)], 1u);
                __syncthreads();
            }
            if (warp == 0) {
                // lane l sums bins [64 l, 64 l + 64); suffix sums over lanes; the
                // lane holding the need-th largest scans its bins from the top
                const int nb = 1 << bits, per = nb / 32;
                uint32_t sl = 0;
                const uint4* h4 = reinterpret_cast<const uint4*>(s_hist + lane * per);
#pragma unroll 4
                for (int e = 0; e < per / 4; ++e) {
                    const uint4 v = h4[e];
                    sl += v.x + v.y + v.z + v.w;
                }
                uint32_t suf = sl;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
                    if (lane + o < 32) suf += y;
                }
                // the lane whose bins hold the need-th largest key; then the whole
                // warp scans that lane's bins (per / 32 each, from the top)
                const uint32_t mine = __ballot_sync(0xffffffffu, suf - sl < need && need <= suf);
                const int L = __ffs(mine) - 1;
                const uint32_t above = __shfl_sync(0xffffffffu, suf - sl, L);   // keys in higher lanes' bins
                const int sub = per / 32;                  // 2 bins per lane (11 bits) or 1 (10 bits)
                const int hi_bin = L * per + per - 1 - lane * sub;   // lane 0 takes the top bins
                uint32_t hs = 0, hb[2] = {0u, 0u};
                for (int e = 0; e < sub; ++e) { hb[e] = s_hist[hi_bin - e]; hs += hb[e]; }
                uint32_t inc = hs;                         // keys in bins >= this lane's lowest bin
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                const uint32_t before = above + inc - hs;  // keys in bins above this lane's
                const uint32_t hit = __ballot_sync(0xffffffffu, before < need && need <= before + hs);
                if (lane == __ffs(hit) - 1) {
                    uint32_t c = before;
                    for (int e = 0; e < sub; ++e) {
                        if (c + hb[e] >= need) {
                            s_misc[0] = (uint32_t)(hi_bin - e);
                            s_misc[1] = need - c;
                            s_misc[7] = hb[e];           // keys in the chosen bin
                            break;
                        }
                        c += hb[e];
                    }
                }
            }
            __syncthreads();
            prefix |= s_misc[0] << shift;
            pmask |= ((1u << bits) - 1u) << shift;
            need = s_misc[1];
            const uint32_t inbin = s_misc[7];
            if (inbin <= (uint32_t)kCand || shift == 0) {
                if (shift == 0) { thr = prefix; break; }   // every bit decided
                // compact the bin's keys (one atomic per warp and slot); one warp
                // searches the bits below
#pragma unroll
                for (int k = 0; k < SLOTS; ++k) {
                    const bool in = tid + NT * k < C && (key[k] & pmask) == prefix;
                    const uint32_t m = __ballot_sync(0xffffffffu, in);
                    if (m == 0u) continue;               // warp-uniform
                    uint32_t at = 0;
                    if (lane == __ffs(m) - 1) at = atomicAdd(&s_misc[2], (uint32_t)__popc(m));
                    at = __shfl_sync(0xffffffffu, at, __ffs(m) - 1);
                    if (in) s_cand[at + __popc(m & lt)] = key[k];
                }
                __syncthreads();
                if (warp == 0) {
                    const uint32_t nc = s_misc[2];
                    uint32_t th = prefix;
                    if (nc <= 128) {
                        // four keys per lane (element i = lane + 32 e, padding 0 below
                        // every key of the bin): a warp bitonic sort, descending,
                        // puts the need-th largest at position need - 1 -- 25
                        // shuffle steps instead of a dependent warp count per bit
                        uint32_t v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[e] = (uint32_t)(lane + 32 * e) < nc ? s_cand[lane + 32 * e] : 0u;
#pragma unroll
                        for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
                            for (int j = k >> 1; j > 0; j >>= 1) {
                                if (j >= 32) {           // partners in the same lane
                                    const int js = j >> 5;
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        if (e & js) continue;
                                        const bool up = ((lane + 32 * e) & k) == 0;
                                        const uint32_t a = v[e], b = v[e | js];
                                        v[e] = up ? max(a, b) : min(a, b);
                                        v[e | js] = up ? min(a, b) : max(a, b);
                                    }
                                } else {
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const uint32_t o = __shfl_xor_sync(0xffffffffu, v[e], j);
                                        const bool up = ((lane + 32 * e) & k) == 0;
                                        const bool lower = (lane & j) == 0;
                                        v[e] = (lower == up) ? max(v[e], o) : min(v[e], o);
                                    }
                                }
                            }
                        }
                        const int pos = (int)need - 1;   // 0 <= pos < nc <= 128
                        const int ps = pos >> 5;
                        const uint32_t mine = ps == 0 ? v[0] : ps == 1 ? v[1] : ps == 2 ? v[2] : v[3];
                        th = __shfl_sync(0xffffffffu, mine, pos & 31);
                    } else {
                        for (int bit = shift - 1; bit >= 0; --bit) {
                            const uint32_t cand = th | (1u << bit);
                            uint32_t c = 0;
                            for (uint32_t e = lane; e < nc; e += 32) c += s_cand[e] >= cand ? 1u : 0u;
                            if (__reduce_add_sync(0xffffffffu, c) >= need) th = cand;
                        }
                    }
                    if (lane == 0) s_misc[3] = th;
                }
                __syncthreads();
                thr = s_misc[3];
                break;
            }
            shift -= pass == 0 ? 11 : 10;
        }
    }

    // ---- keep the keys above thr and the first copies of thr, in index order ----
    // Index order is (slot, warp, lane): per-slot ballots within a warp, and
    // one warp scans the per-(slot, warp) counts into exclusive prefixes.
    uint32_t eqb[SLOTS], gtb[SLOTS], tkb[SLOTS];
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        const bool valid = n > 0 && tid + NT * k < C;
        eqb[k] = __ballot_sync(0xffffffffu, valid && key[k] == thr);
        gtb[k] = __ballot_sync(0xffffffffu, valid && key[k] > thr);
        if (lane == 0) s_cnt[k][warp] = (uint32_t)__popc(eqb[k]) | ((uint32_t)__popc(gtb[k]) << 16);
    }
    __syncthreads();
    const float lse = s_lse;
    // exclusive prefix over the SLOTS * kW counts in (slot, warp) order, in place;
    // the totals land in s_misc[4]
    auto scan_counts = [&]() {
        if (warp == 0) {
            constexpr int E = SLOTS * kW / 32;           // entries per lane
            uint32_t* flat = &s_cnt[0][0];
            uint32_t v[E], sum = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) { v[e] = flat[lane * E + e]; sum += v[e]; }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t run = incl - sum;
#pragma unroll
            for (int e = 0; e < E; ++e) { flat[lane * E + e] = run; run += v[e]; }
            if (lane == 31) s_misc[4] = incl;
        }
        __syncthreads();
    };
    scan_counts();
    // ties are counted in the low 16 bits and keys above thr in the high 16
    // bits of each count, so one scan gives both prefixes
    const uint32_t gt_all = s_misc[4] >> 16;
    const uint32_t need_eq = (uint32_t)n - gt_all;
    bool take[SLOTS];
    uint32_t pos0[SLOTS];   // kept keys before this (slot, warp)
    if ((s_misc[4] & 0xffffu) == need_eq) {
        // every copy of thr is kept (the usual case): the kept keys are those
        // >= thr, and the one scan already counts them
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) {
            tkb[k] = eqb[k] | gtb[k];
            take[k] = (tkb[k] >> lane) & 1u;
            pos0[k] = (s_cnt[k][warp] & 0xffffu) + (s_cnt[k][warp] >> 16);
        }
    } else {
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) {
            const uint32_t rank = (s_cnt[k][warp] & 0xffffu) + __popc(eqb[k] & lt);
            take[k] = ((gtb[k] >> lane) & 1u) || (((eqb[k] >> lane) & 1u) && rank < need_eq);
        }
        __syncthreads();   // s_cnt is rewritten with the kept counts
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) {
            tkb[k] = __ballot_sync(0xffffffffu, take[k]);
            if (lane == 0) s_cnt[k][warp] = (uint32_t)__popc(tkb[k]);
        }
        __syncthreads();
        scan_counts();
#pragma unroll
        for (int k = 0; k < SLOTS; ++k) pos0[k] = s_cnt[k][warp];
    }
    float lse_sel = 0.f;
    if (sh.gate == SAS_GATE_SOFTMAX_SELECTED) {      // normaliser over the kept blocks (CTA-uniform branch)
        float mk = -INFINITY, sk = 0.f;
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (take[k]) mk = fmaxf(mk, xs[k]);
#pragma unroll
        for (int k = 0; k < SLOTS; ++k)
            if (take[k]) sk += expf(xs[k] - mk);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, mk, o), s2 = __shfl_xor_sync(0xffffffffu, sk, o);
            const float mm = fmaxf(mk, m2);
            sk = (mk == -INFINITY ? 0.f : sk * expf(mk - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
            mk = mm;
        }
        if (lane == 0) { s_rm[warp] = mk; s_rs[warp] = sk; }
        __syncthreads();
        float M = -INFINITY, L = 0.f;
        for (int w = 0; w < kW; ++w) M = fmaxf(M, s_rm[w]);
        for (int w = 0; w < kW; ++w) L += s_rm[w] == -INFINITY ? 0.f : s_rs[w] * expf(s_rm[w] - M);
        lse_sel = M + logf(L);
    }
    int32_t* io = idx_out + row * K;
    float* go = gl_out + row * K;
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
        if (take[k]) {
            const uint32_t pos = pos0[k] + __popc(tkb[k] & lt);
            io[pos] = tid + NT * k;
            go[pos] = gate_logit_of(sh.gate, xs[k], lse, lse_sel);
        }
    }
    for (int jj = n + tid; jj < K; jj += NT) { io[jj] = -1; go[jj] = 0.f; }
    if (tid == 0) { lse_out[row] = lse; nsel_out[row] = n; }
}

template <int NT, int SLOTS>
cudaError_t run_topk_cta(const Shape& s, const float* scores, const int32_t* lens, int32_t* idx, float* gl,
                         float* lse, int32_t* nsel, cudaStream_t st) {
    KernelTimer kt("block_topk", st);
    cudaError_t e = launch_pdl(block_topk_cta_kernel<NT, SLOTS>, dim3((unsigned)s.rows()), dim3(NT), 0, st, s, scores,
                               lens, idx, gl, lse, nsel);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

// ------------------------------------------------------------ K1b: bitmap ---

// One CTA per (b, g, tau): OR the tile's selections into a shared row of NB
// words (as 32-bit halves: rows 0-31 and 32-63 of the tile), then store it
// column-major so the backward can walk, per key block, the query tiles that
// kept it.
__global__ void __launch_bounds__(256)
sel_bitmap_T_kernel(Shape sh, const int32_t* __restrict__ idx, const int32_t* __restrict__ nsel,
                    uint64_t* __restrict__ maskT) {
    extern __shared__ unsigned int s_half[];   // [NB][2]
    const int tau = blockIdx.x % sh.nT;
    const int bg = blockIdx.x / sh.nT;
    for (int i = threadIdx.x; i < 2 * sh.NB; i += blockDim.x) s_half[i] = 0u;
    __syncthreads();
    const int64_t row0 = (int64_t)bg * sh.T + (int64_t)tau * sh.bs;
    for (int e = threadIdx.x; e < sh.bs * sh.K; e += blockDim.x) {
        const int r = e / sh.K, slot = e % sh.K;
        const int64_t row = row0 + r;
        if (slot < nsel[row]) {
            const int j = idx[row * sh.K + slot];
            if ((unsigned)j < (unsigned)sh.NB) atomicOr(&s_half[2 * j + (r >> 5)], 1u << (r & 31));
        }
    }
    __syncthreads();
    uint64_t* col = maskT + (int64_t)bg * sh.NB * sh.nT;
    for (int j = threadIdx.x; j < sh.NB; j += blockDim.x)
        col[(int64_t)j * sh.nT + tau] = ((uint64_t)s_half[2 * j + 1] << 32) | s_half[2 * j];
}

}  // namespace

bool topk_row_supported(int64_t max_candidates) { return max_candidates <= 8192; }

cudaError_t launch_block_topk(const Shape& s, const float* scores, const int32_t* lens, int32_t* idx, float* gl,
                              float* lse, int32_t* nsel, cudaStream_t st) {
    const int64_t cmax = ((int64_t)s.q_offset + s.T - 1) / s.bs;
    if (cmax <= 32) return run_topk_warp<1>(s, scores, lens, idx, gl, lse, nsel, st);
    if (cmax <= 128) return run_topk_warp<4>(s, scores, lens, idx, gl, lse, nsel, st);
    if (cmax <= 512) return run_topk_warp<16>(s, scores, lens, idx, gl, lse, nsel, st);
    if (cmax <= 2048) return run_topk_cta<256, 8>(s, scores, lens, idx, gl, lse, nsel, st);
    return run_topk_cta<1024, 8>(s, scores, lens, idx, gl, lse, nsel, st);
}

cudaError_t launch_sel_bitmap_T(const Shape& s, const int32_t* idx, const int32_t* nsel, uint64_t* maskT,
                                cudaStream_t st) {
    const size_t smem = sizeof(uint64_t) * (size_t)s.NB;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(sel_bitmap_T_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (int64_t)s.B * s.Hkv * s.nT;
    KernelTimer kt("sel_bitmap_T", st);
    sel_bitmap_T_kernel<<<(unsigned)grid, 256, smem, st>>>(s, idx, nsel, maskT);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas
