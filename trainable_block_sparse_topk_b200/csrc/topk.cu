// topk.cu -- K1 (gate normaliser + hard top-K per row) and K1b (selection bitmap).
//
// Selection rule (SAS study note 1-2, TopK eq.; arXiv text 3 Preliminaries):
// keep the min(K, C) highest scores among a row's C historical candidates;
// equal scores go to the lower block index; output ascending. The gate
// normaliser is log sum_{i<C} exp s_i (study note 2-1 gate eq.; arXiv text 4,
// normalised gate), and the kept blocks' log-gates are s_i minus it.
//
// Exactness: scores are compared through an order-preserving uint32 key, so the
// K-th largest key is found exactly: by a 32-step bitwise search with
// warp-wide counts when one warp owns the row, by an MSB-first radix select
// (4 passes of 8 bits) when a whole CTA does. The elements above it are kept,
// and the ones equal to it are kept in index order until K are chosen. Each thread owns a contiguous run of
// SLOTS candidates, so index order is (thread, slot) order and two prefix scans
// (one for the ties, one for output positions) place everything.
#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

// Inverse of float_key (-0.0 comes back as +0.0, which compares equal).
__device__ __forceinline__ float key_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// A row is processed by NT threads: one warp (NT == 32, several rows per CTA)
// or the whole CTA (NT > 32, one row per CTA).
template <int NT>
struct RowGroup {
    static constexpr int kWarps = NT / 32;
    // Scratch for cross-warp reductions/scans, per group.
    uint32_t* red;  // kWarps + 2 words

    __device__ __forceinline__ void sync() const {
        if (NT == 32) __syncwarp(); else __syncthreads();
    }
    __device__ __forceinline__ int tid() const { return NT == 32 ? (threadIdx.x & 31) : threadIdx.x; }

    // Exclusive prefix sum over the group in thread order; *total gets the sum.
    __device__ __forceinline__ uint32_t excl_scan(uint32_t x, uint32_t* total) const {
        const int lane = threadIdx.x & 31;
        uint32_t inc = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (NT == 32) {
            *total = __shfl_sync(0xffffffffu, inc, 31);
            return inc - x;
        }
        const int w = threadIdx.x >> 5;
        if (lane == 31) red[w] = inc;
        __syncthreads();
        uint32_t before = 0, tot = 0;
        for (int i = 0; i < kWarps; ++i) {
            uint32_t v = red[i];
            before += (i < w) ? v : 0u;
            tot += v;
        }
        __syncthreads();
        *total = tot;
        return before + inc - x;
    }

    __device__ __forceinline__ float max_all(float x) const {
        x = warp_max(x);
        if (NT == 32) return x;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        float* r = reinterpret_cast<float*>(red);
        if (lane == 0) r[w] = x;
        __syncthreads();
        float m = -INFINITY;
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, r[i]);
        __syncthreads();
        return m;
    }
    __device__ __forceinline__ float sum_all(float x) const {
        x = warp_sum(x);
        if (NT == 32) return x;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        float* r = reinterpret_cast<float*>(red);
        if (lane == 0) r[w] = x;
        __syncthreads();
        float m = 0.f;
        for (int i = 0; i < kWarps; ++i) m += r[i];
        __syncthreads();
        return m;
    }
};

// Find the digit of the `need`-th largest key (1-based) from a 256-bin
// histogram; returns the digit and the rank of that key within its bin.
// Executed by one full warp.
__device__ __forceinline__ void pick_digit(const uint32_t* hist, uint32_t need, uint32_t* digit,
                                           uint32_t* need_in_bin) {
    const int lane = threadIdx.x & 31;
    uint32_t h[8], s8 = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) { h[b] = hist[lane * 8 + b]; s8 += h[b]; }
    // suffix sums over lanes: count in bins >= lane*8
    uint32_t suf = s8;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
    }
    const uint32_t above = suf - s8;
    const bool mine = (above < need) && (need <= suf);
    uint32_t d = 0, nb = 0;
    if (mine) {
        uint32_t c = above;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
            if (d == 0 && nb == 0 && c + h[b] >= need) { d = lane * 8 + b + 1; nb = need - c; }
            c += h[b];
        }
    }
    const uint32_t ball = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(ball) - 1;
    *digit = __shfl_sync(0xffffffffu, d, src) - 1;
    *need_in_bin = __shfl_sync(0xffffffffu, nb, src);
}

template <int NT, int SLOTS>
__global__ void __launch_bounds__(NT == 32 ? 256 : NT)
block_topk_kernel(Shape sh, const float* __restrict__ scores, int32_t* __restrict__ idx_out,
                  float* __restrict__ gl_out, float* __restrict__ lse_out, int32_t* __restrict__ nsel_out) {
    constexpr int kRowsPerCta = NT == 32 ? 8 : 1;
    constexpr int kWarps = NT / 32;
    __shared__ uint32_t s_hist[kRowsPerCta][256];
    __shared__ uint32_t s_red[kRowsPerCta][kWarps + 4];

    const int grp = NT == 32 ? (threadIdx.x >> 5) : 0;
    const int64_t row = (int64_t)blockIdx.x * kRowsPerCta + grp;
    const bool row_ok = row < sh.rows();   // uniform per group
    RowGroup<NT> G{s_red[grp]};
    const int tid = G.tid();
    uint32_t* hist = s_hist[grp];

    const int t = row_ok ? (int)(row % sh.T) : 0;
    const int64_t p = (int64_t)sh.q_offset + t;
    const int C = row_ok ? (int)(p / sh.bs) : 0;
    const int K = sh.K;
    const int n = C < K ? C : K;
    const float* srow = scores + row * sh.NB;

    // --- load keys (thread owns candidates [tid*SLOTS, tid*SLOTS + SLOTS)) ---
    uint32_t key[SLOTS];
    float mloc = -INFINITY;
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        const int i = tid * SLOTS + j;
        if (i < C) {
            const float f = srow[i];
            key[j] = float_key(f);
            mloc = fmaxf(mloc, f);
        } else {
            key[j] = 0u;  // below every valid key (float_key(-inf) = 0x007fffff)
        }
    }

    // --- gate normaliser: lse = m + log sum exp(s - m) ---
    const float m = G.max_all(mloc);
    float lsum = 0.f;
    if (m != -INFINITY) {
#pragma unroll
        for (int j = 0; j < SLOTS; ++j)
            if (tid * SLOTS + j < C) lsum += expf(key_float(key[j]) - m);
    }
    lsum = G.sum_all(lsum);
    const float lse = (C > 0 && m != -INFINITY) ? m + logf(lsum) : -INFINITY;

    // --- the n-th largest key ---
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)n;
    if (NT == 32 && n > 0) {
        // One warp: bitwise search, MSB first. Bit b joins the answer when at
        // least n keys are >= (answer | bit): the result is the largest v with
        // #{keys >= v} >= n, i.e. the n-th largest key. Invalid slots hold key
        // 0, which no candidate (>= 1) admits.
        uint32_t thr = 0;
#pragma unroll
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t cand = thr | (1u << bit);
            uint32_t c = 0;
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) c += key[j] >= cand ? 1u : 0u;
            if (__reduce_add_sync(0xffffffffu, c) >= (uint32_t)n) thr = cand;
        }
        uint32_t gt = 0;
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) gt += key[j] > thr ? 1u : 0u;
        prefix = thr;
        need = (uint32_t)n - __reduce_add_sync(0xffffffffu, gt);   // copies of thr to keep
    } else if (n > 0) {
        // radix select, 4 passes of 8 bits, MSB first
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int b = tid; b < 256; b += NT) hist[b] = 0;
            G.sync();
#pragma unroll
            for (int j = 0; j < SLOTS; ++j) {
                const bool act = (tid * SLOTS + j < C) && ((key[j] & pmask) == prefix);
                const uint32_t bin = (key[j] >> shift) & 255u;
                const uint32_t peers = __match_any_sync(0xffffffffu, act ? bin : 0xffffffffu);
                if (act && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
            }
            G.sync();
            uint32_t dgt, nb;
            if (NT == 32) {
                pick_digit(hist, need, &dgt, &nb);
            } else {
                if (threadIdx.x < 32) {
                    pick_digit(hist, need, &dgt, &nb);
                    if (threadIdx.x == 0) { s_red[grp][kWarps] = dgt; s_red[grp][kWarps + 1] = nb; }
                }
                __syncthreads();
                dgt = s_red[grp][kWarps];
                nb = s_red[grp][kWarps + 1];
                __syncthreads();
            }
            prefix |= dgt << shift;
            pmask |= 255u << shift;
            need = nb;
        }
    }
    const uint32_t thr = prefix;   // the n-th largest key; `need` of its copies are kept

    // --- ties: keep the first `need` elements equal to thr, in index order ---
    uint32_t eq_loc = 0;
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) eq_loc += (n > 0 && tid * SLOTS + j < C && key[j] == thr) ? 1u : 0u;
    uint32_t tot;
    uint32_t eq_before = G.excl_scan(eq_loc, &tot);
    uint32_t take_mask = 0, take_loc = 0;
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        const bool valid = n > 0 && tid * SLOTS + j < C;
        bool take = valid && key[j] > thr;
        if (valid && key[j] == thr) {
            take = eq_before < need;
            ++eq_before;
        }
        if (take) { take_mask |= 1u << j; ++take_loc; }
    }
    uint32_t pos = G.excl_scan(take_loc, &tot);

    if (!row_ok) return;
    int32_t* io = idx_out + row * K;
    float* go = gl_out + row * K;
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) {
        if (take_mask & (1u << j)) {
            const int i = tid * SLOTS + j;
            io[pos] = i;
            go[pos] = sh.gate == SAS_GATE_SOFTMAX ? key_float(key[j]) - lse : 0.f;
            ++pos;
        }
    }
    for (int jj = n + tid; jj < K; jj += NT) { io[jj] = -1; go[jj] = 0.f; }
    if (tid == 0) { lse_out[row] = lse; nsel_out[row] = n; }
}

template <int NT, int SLOTS>
cudaError_t run_topk(const Shape& s, const float* scores, int32_t* idx, float* gl, float* lse, int32_t* nsel,
                     cudaStream_t st) {
    const int64_t rows = s.rows();
    const int rpc = NT == 32 ? 8 : 1;
    const int64_t grid = (rows + rpc - 1) / rpc;
    KernelTimer kt("block_topk", st);
    block_topk_kernel<NT, SLOTS><<<(unsigned)grid, NT == 32 ? 256 : NT, 0, st>>>(s, scores, idx, gl, lse, nsel);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

// ------------------------------------------------------------ K1b: bitmap ---

// One CTA per (b, g, tau): OR the tile's selections into a shared row of NB
// words, then store it column-major so the backward can walk, per key block,
// the query tiles that kept it.
__global__ void __launch_bounds__(256)
sel_bitmap_T_kernel(Shape sh, const int32_t* __restrict__ idx, const int32_t* __restrict__ nsel,
                    uint64_t* __restrict__ maskT) {
    extern __shared__ unsigned long long s_words[];
    const int tau = blockIdx.x % sh.nT;
    const int bg = blockIdx.x / sh.nT;
    for (int j = threadIdx.x; j < sh.NB; j += blockDim.x) s_words[j] = 0ull;
    __syncthreads();
    const int64_t row0 = (int64_t)bg * sh.T + (int64_t)tau * sh.bs;
    for (int e = threadIdx.x; e < sh.bs * sh.K; e += blockDim.x) {
        const int r = e / sh.K, slot = e % sh.K;
        const int64_t row = row0 + r;
        if (slot < nsel[row]) {
            const int j = idx[row * sh.K + slot];
            if ((unsigned)j < (unsigned)sh.NB) atomicOr(&s_words[j], 1ull << r);
        }
    }
    __syncthreads();
    uint64_t* col = maskT + (int64_t)bg * sh.NB * sh.nT;
    for (int j = threadIdx.x; j < sh.NB; j += blockDim.x) col[(int64_t)j * sh.nT + tau] = s_words[j];
}

}  // namespace

bool topk_row_supported(int64_t max_candidates) { return max_candidates <= 8192; }

cudaError_t launch_block_topk(const Shape& s, const float* scores, int32_t* idx, float* gl, float* lse,
                              int32_t* nsel, cudaStream_t st) {
    const int64_t cmax = ((int64_t)s.q_offset + s.T - 1) / s.bs;
    if (cmax <= 32) return run_topk<32, 1>(s, scores, idx, gl, lse, nsel, st);
    if (cmax <= 128) return run_topk<32, 4>(s, scores, idx, gl, lse, nsel, st);
    if (cmax <= 512) return run_topk<32, 16>(s, scores, idx, gl, lse, nsel, st);
    if (cmax <= 2048) return run_topk<256, 8>(s, scores, idx, gl, lse, nsel, st);
    return run_topk<1024, 8>(s, scores, idx, gl, lse, nsel, st);
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
