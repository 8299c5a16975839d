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
// Each CTA scores kTile blocks of one (b, g) row; half a warp reads one
// 256-byte pooled key with 16-byte loads (two keys per warp instruction) and
// reduces its dot product with shuffles.
#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 256;   // blocks per CTA
constexpr int kD = 128;

__global__ void __launch_bounds__(kThreads)
pooled_score_kernel(Shape sh, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kbar,
                    int64_t kstride, float* __restrict__ scores) {
    pdl_trigger();   // the top-K after this kernel waits for its end before reading the scores
    const int tiles = (sh.NB + kTile - 1) / kTile;
    const int64_t bg = blockIdx.x / tiles;
    const int tile = (int)(blockIdx.x - bg * tiles);
    const int b = (int)(bg / sh.Hkv), g = (int)(bg - (int64_t)b * sh.Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, c = lane & 15;            // 16 lanes per pooled key, 8 dims each
    const int C = (int)(sh.q_offset / sh.bs);
    // this lane's 8 dims of qbar
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
    const __nv_bfloat16* kr = kbar + (int64_t)bg * kstride * kD;
    float* sr = scores + (int64_t)bg * sh.NB;
    const int j0 = tile * kTile;
#pragma unroll 4
    for (int jj = warp * 2 + half; jj < kTile; jj += 2 * (kThreads / 32)) {
        const int j = j0 + jj;
        float acc = 0.f;
        if (j < C) {
            float x[8];
            load_vec<__nv_bfloat16, 8>(kr + (int64_t)j * kD + c * 8, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(qb[e], x[e], acc);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (c == 0 && j < sh.NB) sr[j] = acc;
    }
}

}  // namespace

cudaError_t launch_pooled_scores(const Shape& s, const void* q, const void* kbar, int64_t kstride, float* scores,
                                 cudaStream_t st) {
    if (s.dtype != SAS_DT_BF16 || s.D != kD) return cudaErrorInvalidValue;
    const int tiles = (s.NB + kTile - 1) / kTile;
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
