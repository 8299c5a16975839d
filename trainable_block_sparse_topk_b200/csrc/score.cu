// score.cu -- block scores of decode rows from pooled keys.
//
// Before the top-K, the serving path scores every cached block of the new
// token's KV group (SAS study note 3-7 inference path, step 1; at long
// context this scan dominates the decode step, study note 5-6). The selector
// of the pages is a trained network; the fixed scorer here stands in for it:
//   s[b, g, 0, j] = qbar . kbar[b, g, j],  j < C = floor(q_offset / block),
// with qbar the mean of the group's G query heads and kbar[b, g, j] the mean
// key of block j, kept by the caller beside the cache. Columns j >= C are 0.
//
// The scan reads B * Hkv * C pooled keys of d bf16 values once: HBM-bound.
// Each CTA scores kKeys consecutive blocks of one (b, g) row: one bulk copy
// brings their pooled keys (32 KiB, contiguous) into shared memory while the
// threads form qbar, then half a warp dots one 256-byte key (16-byte reads,
// two keys per warp instruction) and reduces with shuffles. Seven such CTAs
// fit on an SM, so ~224 KiB per SM are in flight without holding registers.
#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

constexpr int kThreads = 256;
constexpr int kKeys = 128;   // blocks per CTA
constexpr int kD = 128;

__global__ void __launch_bounds__(kThreads)
pooled_score_kernel(Shape sh, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kbar,
                    int64_t kstride, float* __restrict__ scores) {
    __shared__ __align__(128) uint4 s_k[kKeys * (kD * 2 / 16)];
    __shared__ __align__(8) uint64_t s_bar;
    pdl_trigger();   // the top-K after this kernel waits for its end before reading the scores
    const int tiles = (sh.NB + kKeys - 1) / kKeys;
    const int64_t bg = blockIdx.x / tiles;
    const int tile = (int)(blockIdx.x - bg * tiles);
    const int b = (int)(bg / sh.Hkv), g = (int)(bg - (int64_t)b * sh.Hkv);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = lane >> 4, c = lane & 15;            // 16 lanes per pooled key, 8 dims each
    const int C = (int)(sh.q_offset / sh.bs);
    const int j0 = tile * kKeys;
    const int nk = max(0, min(kKeys, C - j0));            // keys of this tile with a score to compute
    const __nv_bfloat16* kr = kbar + sh.kv_index(bg) * kstride * kD;   // pooled keys of the KV head
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0 && nk > 0) {
        mbar_arrive_expect_tx(&s_bar, (uint32_t)nk * kD * 2);
        bulk_g2s(s_k, kr + (int64_t)j0 * kD, (uint32_t)nk * kD * 2, &s_bar);
    }
    // this lane's 8 dims of qbar, while the keys are on their way
    float qb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int h = 0; h < sh.G; ++h) {
        float x[8];
        load_vec<__nv_bfloat16, 8>(q + ((int64_t)b * sh.Hq + (int64_t)g * sh.G + h) * kD + c * 8, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) qb[e] += x[e];
    }
    const float inv = 1.f / (float)sh.G;
#pragma unroll
    for (int e = 0; e < 8; ++e) qb[e] *= inv;
    bool ok = true;
    if (nk > 0) {
        ok = mbar_wait_bounded(&s_bar, 0u);
        // a copy that has not landed by the limit may still write: let it land
        // (bounded) before the CTA exits
        if (!ok && tid == 0) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(&s_bar, 0u) && global_ns() - t0 < kDefaultWaitNs) {
            }
        }
    }
    float* sr = scores + (int64_t)bg * sh.NB;
#pragma unroll 4
    for (int jj = warp * 2 + half; jj < kKeys; jj += 2 * (kThreads / 32)) {
        const int j = j0 + jj;
        float acc = 0.f;
        if (jj < nk) {
            const uint4 raw = s_k[jj * (kD * 2 / 16) + c];
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                acc = fmaf(qb[2 * e], f.x, acc);
                acc = fmaf(qb[2 * e + 1], f.y, acc);
            }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (!ok) acc = __int_as_float(0x7fc00000);
        if (c == 0 && j < sh.NB) sr[j] = acc;
    }
}

}  // namespace

cudaError_t launch_pooled_scores(const Shape& s, const void* q, const void* kbar, int64_t kstride, float* scores,
                                 cudaStream_t st) {
    if (s.dtype != SAS_DT_BF16 || s.D != kD) return cudaErrorInvalidValue;
    const int tiles = (s.NB + kKeys - 1) / kKeys;
    const int64_t grid = (int64_t)s.B * s.Hkv * tiles;
    {
        KernelTimer kt("pooled_score", st);
        pooled_score_kernel<<<(unsigned)grid, kThreads, 0, st>>>(s, static_cast<const __nv_bfloat16*>(q),
                                                                 static_cast<const __nv_bfloat16*>(kbar), kstride,
                                                                 scores);
    }
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas
