// attn_simt.cu -- gated block-sparse attention on CUDA cores (exact fp32 math).
//
// This path serves the fp32 dtype (no TF32 anywhere, for 1e-4 parity) and any
// shape the tensor-core kernels do not take. Its arithmetic follows the
// method's definition (SAS study note 2-2 gated-attention eq.; arXiv text 4):
//   a_j = scale * q . k_j + log g_blk(j)   over the kept blocks' tokens,
//   a_j = scale * q . k_j                  over the current block, j <= p,
//   o = softmax(a) V,
// and the backward recomputes P = exp(a - lse):
//   dV_j += P_j dO, dP_j = dO . v_j, dS_j = P_j (dP_j - D), D = dO . o,
//   dQ = scale sum_j dS_j k_j, dK_j += scale dS_j q,
//   Gsum[row, slot] = sum over the G heads and the block's tokens of dS
// (the gradient w.r.t. the block's log-gate, study note 3-6 "keeps the
// selector gradient").
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

// ------------------------------------------------------------------ forward ---

template <typename T, int D, int GMAX, int BS>
__device__ __forceinline__ void fwd_simt_row(const Shape& sh, const T* __restrict__ q, const T* __restrict__ k,
                                             const T* __restrict__ v, const int32_t* __restrict__ idx,
                                             const float* __restrict__ gl, const int32_t* __restrict__ nsel,
                                             T* __restrict__ o, float* __restrict__ attn_lse, int64_t row,
                                             float (*s_qw)[D], float (*s_pw)[GMAX], int lane);

// One warp per (b, kv head, t) row, all G heads of the group at once. Lane
// `l` scores keys l and l + 32 of each kept block and owns D/32 output dims.
// With `list` set, the warps instead stride over the rows list[0 .. *list_n)
// (recomputing rows another kernel flagged); otherwise warp w of block x takes
// row 4 x + w.
template <typename T, int D, int GMAX, int BS>
__global__ void __launch_bounds__(128)
fwd_simt_kernel(Shape sh, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const int32_t* __restrict__ idx, const float* __restrict__ gl,
                const int32_t* __restrict__ nsel, T* __restrict__ o, float* __restrict__ attn_lse,
                const int32_t* __restrict__ list, const int32_t* __restrict__ list_n) {
    constexpr int W = 4;
    __shared__ float s_q[W][GMAX][D];
    __shared__ float s_p[W][BS][GMAX];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (list != nullptr) {
        const int n = *list_n;
        for (int i = (int)blockIdx.x * W + w; i < n; i += (int)gridDim.x * W)
            fwd_simt_row<T, D, GMAX, BS>(sh, q, k, v, idx, gl, nsel, o, attn_lse, list[i], s_q[w], s_p[w], lane);
        return;
    }
    const int64_t row = (int64_t)blockIdx.x * W + w;
    if (row >= sh.rows()) return;
    fwd_simt_row<T, D, GMAX, BS>(sh, q, k, v, idx, gl, nsel, o, attn_lse, row, s_q[w], s_p[w], lane);
}

template <typename T, int D, int GMAX, int BS>
__device__ __forceinline__ void fwd_simt_row(const Shape& sh, const T* __restrict__ q, const T* __restrict__ k,
                                             const T* __restrict__ v, const int32_t* __restrict__ idx,
                                             const float* __restrict__ gl, const int32_t* __restrict__ nsel,
                                             T* __restrict__ o, float* __restrict__ attn_lse, int64_t row,
                                             float (*s_qw)[D], float (*s_pw)[GMAX], int lane) {
    constexpr int KPL = BS / 32;
    constexpr int DPL = D / 32;
    constexpr int V16 = vec16<T>();
    const int G = sh.G;
    const int64_t bg = row / sh.T;
    const int t = (int)(row % sh.T);
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int C = t / BS;
    const int n = nsel[row];
    const float qscale = sh.scale * kLog2e;   // logits in log2 units

#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        if (h < G) {
            const T* qh = q + (((int64_t)b * sh.Hq + g * G + h) * sh.T + t) * D;
            for (int d = lane; d < D; d += 32) s_qw[h][d] = Elem<T>::to_f(qh[d]) * qscale;
        }
    }
    __syncwarp();

    float m[GMAX], l[GMAX], acc[GMAX][DPL];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
    }
    const T* kb = k + sh.kv_index(bg) * (int64_t)sh.T * D;
    const T* vb = v + sh.kv_index(bg) * (int64_t)sh.T * D;

    for (int jj = 0; jj <= n; ++jj) {
        const bool hist = jj < n;
        const int j = hist ? idx[row * sh.K + jj] : C;
        const float lg = hist ? gl[row * sh.K + jj] * kLog2e : 0.f;
        const int ntok = hist ? BS : (t - C * BS + 1);
        if ((unsigned)j > (unsigned)C) continue;   // not a valid selection: skipped, never read

        float sc[KPL][GMAX];
#pragma unroll
        for (int kk = 0; kk < KPL; ++kk) {
            const int key = lane + 32 * kk;
#pragma unroll
            for (int h = 0; h < GMAX; ++h) sc[kk][h] = 0.f;
            if (key < ntok) {
                const T* kr = kb + ((int64_t)j * BS + key) * D;
#pragma unroll 4
                for (int c = 0; c < D / V16; ++c) {
                    float kv[V16];
                    load_vec<T, V16>(kr + c * V16, kv);
#pragma unroll
                    for (int h = 0; h < GMAX; ++h) {
                        if (h < G) {
#pragma unroll
                            for (int e = 0; e < V16; ++e) sc[kk][h] = fmaf(s_qw[h][c * V16 + e], kv[e], sc[kk][h]);
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < GMAX; ++h) sc[kk][h] += lg;
            } else {
#pragma unroll
                for (int h = 0; h < GMAX; ++h) sc[kk][h] = -INFINITY;
            }
        }
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h >= G) continue;
            float mx = sc[0][h];
#pragma unroll
            for (int kk = 1; kk < KPL; ++kk) mx = fmaxf(mx, sc[kk][h]);
            mx = warp_max(mx);
            const float mn = fmaxf(m[h], mx);
            const float corr = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - mn);
            float ps = 0.f;
#pragma unroll
            for (int kk = 0; kk < KPL; ++kk) {
                const float pk = (mn == -INFINITY) ? 0.f : exp2f(sc[kk][h] - mn);
                s_pw[lane + 32 * kk][h] = pk;
                ps += pk;
            }
            ps = warp_sum(ps);
            l[h] = l[h] * corr + ps;
            m[h] = mn;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] *= corr;
        }
        __syncwarp();
        for (int key = 0; key < ntok; ++key) {
            float vv[DPL];
            load_vec<T, DPL>(vb + ((int64_t)j * BS + key) * D + lane * DPL, vv);
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                if (h < G) {
                    const float pk = s_pw[key][h];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pk, vv[e], acc[h][e]);
                }
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        if (h >= G) continue;
        const int64_t orow = ((int64_t)b * sh.Hq + g * G + h) * sh.T + t;
        const float inv = 1.f / l[h];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[orow * D + lane * DPL + e] = Elem<T>::from_f(acc[h][e] * inv);
        if (lane == 0) attn_lse[orow] = (m[h] + log2f(l[h])) * kLn2;
    }
}

// ---------------------------------------------------------- D = rowsum(dO*O) ---

// D = rowsum(o * dO) per query-head row. A row is read by D / V lanes with
// 16-byte loads (V elements each), so one warp instruction covers 32 V / D
// rows; each warp issues kU such instructions for both tensors before it
// reduces any, keeping 32 16-byte loads per thread in flight. The same lanes
// zero the row of the fp32 dq accumulator (D floats) that the backward adds
// into.
template <typename T>
__device__ __forceinline__ float dot16(const uint4& x, const uint4& y) {
    float ax[vec16<T>()], ay[vec16<T>()];
    load_vec<T, vec16<T>()>(reinterpret_cast<const T*>(&x), ax);
    load_vec<T, vec16<T>()>(reinterpret_cast<const T*>(&y), ay);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < vec16<T>(); ++e) s = fmaf(ax[e], ay[e], s);
    return s;
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
rowdot_kernel(int64_t rows, const T* __restrict__ o, const T* __restrict__ dO, float* __restrict__ Dd,
              float* __restrict__ dq_acc) {
    constexpr int V = vec16<T>();
    constexpr int LPR = D / V;          // lanes per row
    constexpr int RPI = 32 / LPR;       // rows per warp instruction
    constexpr int kU = 4;
    constexpr int RW = RPI * kU;        // rows per warp pass
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = warp * RW; r0 < rows; r0 += nwarps * RW) {   // warp-uniform
        uint4 x[kU], y[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t row = r0 + u * RPI + sub;
            x[u] = y[u] = make_uint4(0u, 0u, 0u, 0u);
            if (row < rows) {
                x[u] = *reinterpret_cast<const uint4*>(o + row * D + li * V);
                y[u] = *reinterpret_cast<const uint4*>(dO + row * D + li * V);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float sum = dot16<T>(x[u], y[u]);
#pragma unroll
            for (int m = LPR / 2; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
            const int64_t row = r0 + u * RPI + sub;
            if (li == 0 && row < rows) Dd[row] = sum;
            if (row < rows) {
                float4* z = reinterpret_cast<float4*>(dq_acc + row * D + li * V);
#pragma unroll
                for (int e = 0; e < V / 4; ++e) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
}

// ----------------------------------------------------------------- backward ---

// One CTA per (b, kv head, key block j), 4 threads per key. It visits every
// query that attends block j: all of tile j (the block is their current block,
// causal) and, from the column bitmap, each later query that kept j. dK_j and
// dV_j accumulate in registers; dQ goes to an fp32 buffer by atomic add; the
// per-(row, slot) log-gate gradient Gsum is summed over the G heads here.
template <typename T, int D, int GMAX, int BS>
__global__ void __launch_bounds__(BS * 4)
bwd_simt_kernel(Shape sh, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const T* __restrict__ dO, const float* __restrict__ attn_lse, const float* __restrict__ Dd,
                const int32_t* __restrict__ idx, const float* __restrict__ gl, const int32_t* __restrict__ nsel,
                const uint64_t* __restrict__ maskT, float* __restrict__ dq_acc, T* __restrict__ dk,
                T* __restrict__ dv, float* __restrict__ dk32, float* __restrict__ dv32, float* __restrict__ gsum) {
    constexpr int NT = BS * 4;
    constexpr int DS = D + 4;          // padded row stride: conflict-free for (kk, qd) threads
    constexpr int DQ = D / 4;
    extern __shared__ float smem[];
    float* Ks = smem;                  // [BS][DS]
    float* Vs = Ks + BS * DS;          // [BS][DS]
    float* qs = Vs + BS * DS;          // [GMAX][D]
    float* dOs = qs + GMAX * D;        // [GMAX][D]
    float* dSs = dOs + GMAX * D;       // [GMAX][BS]
    float* st = dSs + GMAX * BS;       // [2][GMAX]: lse, D
    float* red = st + 2 * GMAX;        // [NT/32]

    const int G = sh.G;
    const int j = blockIdx.x % sh.nT;
    const int64_t bg = blockIdx.x / sh.nT;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int tid = threadIdx.x;
    const int kk = tid >> 2, qd = tid & 3;
    const float scale = sh.scale;

    const T* kb = k + (sh.kv_index(bg) * sh.T + (int64_t)j * BS) * D;
    const T* vb = v + (sh.kv_index(bg) * sh.T + (int64_t)j * BS) * D;
    for (int e = tid; e < BS * D; e += NT) {
        Ks[(e / D) * DS + e % D] = Elem<T>::to_f(kb[e]);
        Vs[(e / D) * DS + e % D] = Elem<T>::to_f(vb[e]);
    }
    float dk_r[DQ], dv_r[DQ];
#pragma unroll
    for (int i = 0; i < DQ; ++i) { dk_r[i] = 0.f; dv_r[i] = 0.f; }
    __syncthreads();

    const uint64_t* col = maskT + (bg * sh.NB + j) * (int64_t)sh.nT;

    // Token stream: tile j fully (diagonal), then set bits of later tiles.
    int tau = j;
    uint64_t word = (BS == 64) ? ~0ull : ((1ull << BS) - 1ull);
    while (true) {
        if (word == 0ull) {
            if (++tau >= sh.nT) break;
            word = col[tau];
            continue;
        }
        const int r = __ffsll((long long)word) - 1;
        word &= word - 1ull;
        const bool diag = tau == j;
        const int t = tau * BS + r;
        const int64_t row = bg * sh.T + t;
        int slot = -1;
        float lg = 0.f;
        if (!diag) {
            // position of j in the row's ascending kept list
            const int32_t* ir = idx + row * sh.K;
            int lo = 0, hi = nsel[row] - 1;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (ir[mid] < j) lo = mid + 1; else hi = mid;
            }
            slot = lo;
            lg = gl[row * sh.K + slot];
        }
        const int kmax = diag ? r : BS - 1;   // causal limit inside the current block

        for (int e = tid; e < G * D; e += NT) {
            const int h = e / D, d = e % D;
            const int64_t qrow = ((int64_t)b * sh.Hq + g * G + h) * sh.T + t;
            qs[h * D + d] = Elem<T>::to_f(q[qrow * D + d]);
            dOs[h * D + d] = Elem<T>::to_f(dO[qrow * D + d]);
        }
        if (tid < G) {
            const int64_t qrow = ((int64_t)b * sh.Hq + g * G + tid) * sh.T + t;
            st[tid] = attn_lse[qrow];
            st[GMAX + tid] = Dd[qrow];
        }
        __syncthreads();

#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h >= G) continue;
            float sd = 0.f, pd = 0.f;
#pragma unroll
            for (int i = 0; i < DQ; ++i) {
                sd = fmaf(qs[h * D + qd + 4 * i], Ks[kk * DS + qd + 4 * i], sd);
                pd = fmaf(dOs[h * D + qd + 4 * i], Vs[kk * DS + qd + 4 * i], pd);
            }
            sd += __shfl_xor_sync(0xffffffffu, sd, 1);
            sd += __shfl_xor_sync(0xffffffffu, sd, 2);
            pd += __shfl_xor_sync(0xffffffffu, pd, 1);
            pd += __shfl_xor_sync(0xffffffffu, pd, 2);
            const float P = (kk <= kmax) ? expf(scale * sd + lg - st[h]) : 0.f;
            const float dS = P * (pd - st[GMAX + h]);
#pragma unroll
            for (int i = 0; i < DQ; ++i) {
                dv_r[i] = fmaf(P, dOs[h * D + qd + 4 * i], dv_r[i]);
                dk_r[i] = fmaf(scale * dS, qs[h * D + qd + 4 * i], dk_r[i]);
            }
            if (qd == 0) dSs[h * BS + kk] = dS;
        }
        __syncthreads();

        for (int e = tid; e < G * D; e += NT) {
            const int h = e / D, d = e % D;
            float a = 0.f;
#pragma unroll 8
            for (int x = 0; x < BS; ++x) a = fmaf(dSs[h * BS + x], Ks[x * DS + d], a);
            const int64_t qrow = ((int64_t)b * sh.Hq + g * G + h) * sh.T + t;
            atomicAdd(&dq_acc[qrow * D + d], scale * a);
        }
        if (!diag) {
            float a = 0.f;
            for (int e = tid; e < G * BS; e += NT) a += dSs[e];
            a = warp_sum(a);
            if ((tid & 31) == 0) red[tid >> 5] = a;
        }
        __syncthreads();
        if (!diag && tid == 0) {
            float a = 0.f;
            for (int w = 0; w < NT / 32; ++w) a += red[w];
            gsum[row * sh.K + slot] = a;
        }
    }

    // per-query-head selection: fp32 partials of this selection group, summed
    // over the heads of the KV head afterwards
    const int64_t kv0 = (bg * sh.T + (int64_t)j * BS) * D;
#pragma unroll
    for (int i = 0; i < DQ; ++i) {
        const int64_t at = kv0 + kk * D + qd + 4 * i;
        if (dk32 != nullptr) {
            dk32[at] = dk_r[i];
            dv32[at] = dv_r[i];
        } else {
            dk[at] = Elem<T>::from_f(dk_r[i]);
            dv[at] = Elem<T>::from_f(dv_r[i]);
        }
    }
}

// Per-query-head selection: dK, dV of KV head kv = the sum of the fp32
// partials of its kvdiv query heads (selection groups kv * kvdiv + r), one
// float4 per thread and pass.
template <typename T>
__global__ void __launch_bounds__(256)
reduce_dkv_kernel(Shape sh, const float* __restrict__ dk32, const float* __restrict__ dv32, T* __restrict__ dk,
                  T* __restrict__ dv) {
    const int64_t per = (int64_t)sh.T * sh.D / 4;              // float4s per (b, kv head)
    const int64_t n = (int64_t)sh.B * sh.Hkvp * per;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bk = i / per, e = i - bk * per;
        const int64_t b = bk / sh.Hkvp, kv = bk - b * sh.Hkvp;
        float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
        for (int r = 0; r < sh.kvdiv; ++r) {
            const int64_t src = (b * sh.Hkv + kv * sh.kvdiv + r) * per + e;
            const float4 a = reinterpret_cast<const float4*>(dk32)[src];
            const float4 c = reinterpret_cast<const float4*>(dv32)[src];
            sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
            sv.x += c.x; sv.y += c.y; sv.z += c.z; sv.w += c.w;
        }
        T* ok = dk + i * 4;
        T* ov = dv + i * 4;
        ok[0] = Elem<T>::from_f(sk.x); ok[1] = Elem<T>::from_f(sk.y); ok[2] = Elem<T>::from_f(sk.z); ok[3] = Elem<T>::from_f(sk.w);
        ov[0] = Elem<T>::from_f(sv.x); ov[1] = Elem<T>::from_f(sv.y); ov[2] = Elem<T>::from_f(sv.z); ov[3] = Elem<T>::from_f(sv.w);
    }
}

// fp32 -> bf16, 8 values per thread and pass, two passes' loads in flight
// (n8 = number of 8-value groups).
__global__ void __launch_bounds__(256)
cast_bf16x8_kernel(int64_t n8, const float4* __restrict__ src, uint4* __restrict__ dst, const int* __restrict__ aborted) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (aborted != nullptr && *aborted) {   // the accumulator is incomplete: mark dq invalid
        const uint32_t nan2 = 0x7fc07fc0u;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride)
            dst[i] = make_uint4(nan2, nan2, nan2, nan2);
        return;
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += 2 * stride) {
        float4 v[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t k = i + u * stride;
            if (k < n8) {
                v[u][0] = src[2 * k];
                v[u][1] = src[2 * k + 1];
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t k = i + u * stride;
            if (k >= n8) continue;
            __nv_bfloat162 p[4] = {__floats2bfloat162_rn(v[u][0].x, v[u][0].y), __floats2bfloat162_rn(v[u][0].z, v[u][0].w),
                                   __floats2bfloat162_rn(v[u][1].x, v[u][1].y), __floats2bfloat162_rn(v[u][1].z, v[u][1].w)};
            dst[k] = *reinterpret_cast<const uint4*>(p);
        }
    }
}

// ------------------------------------------------------- score gradient (K5) ---

// The kept blocks' own terms kv[r] (slots lane and lane + 32; si[r] = -1 when
// not kept) and the factor T of the dense term -g_i T, per gate activation
// (Gsum_k = dL / d log g_k):
//   softmax           d log g_i/ds_k = [i=k] - g_k:  kept Gsum_k, T = sum Gsum
//   sigmoid           log g_k = log sigmoid(s_k):     kept Gsum_k (1 - sigmoid(s_k))
//   raw               log g_k = s_k:                  kept Gsum_k
//   softmax (kept)    log g_k = s_k - log sum_I e^s:  kept Gsum_k - p_k sum Gsum
//   hard (STE)        dL/dg_k = Gsum_k, dg_i/ds_k = g_i([i=k] - g_k):
//                                                     kept Gsum_k g_k, T = sum Gsum g
__device__ __forceinline__ void dscore_kept_terms(int mode, const int (&si)[2], const float (&sg)[2],
                                                  const float (&sk)[2], float lse, float (&kv)[2], float& T) {
    kv[0] = kv[1] = 0.f;
    T = 0.f;
    if (mode == SAS_GATE_SOFTMAX) {
        kv[0] = sg[0];
        kv[1] = sg[1];
        T = warp_sum(sg[0] + sg[1]);
    } else if (mode == SAS_GATE_STE) {
#pragma unroll
        for (int r = 0; r < 2; ++r) kv[r] = si[r] >= 0 ? sg[r] * expf(sk[r] - lse) : 0.f;
        T = warp_sum(kv[0] + kv[1]);
    } else if (mode == SAS_GATE_SIGMOID) {
#pragma unroll
        for (int r = 0; r < 2; ++r) kv[r] = si[r] >= 0 ? sg[r] / (1.f + expf(sk[r])) : 0.f;   // 1 - sigmoid(s)
    } else if (mode == SAS_GATE_RAW) {
        kv[0] = sg[0];
        kv[1] = sg[1];
    } else if (mode == SAS_GATE_SOFTMAX_SELECTED) {
        const float m = warp_max(fmaxf(sk[0], sk[1]));
        const float l = warp_sum((si[0] >= 0 ? expf(sk[0] - m) : 0.f) + (si[1] >= 0 ? expf(sk[1] - m) : 0.f));
        const float tot = warp_sum(sg[0] + sg[1]);
#pragma unroll
        for (int r = 0; r < 2; ++r) kv[r] = si[r] >= 0 ? sg[r] - expf(sk[r] - m) / l * tot : 0.f;
    }
}

// ds_i = dL/ds_i for i < C, 0 otherwise, from Gsum_k = dL/d(log g_k) of the
// kept blocks through the gate activation's derivative. Softmax gate
// (arXiv text 4: d log g_i / d s_k = [i=k] - g_k, g_i = exp(s_i - score_lse)):
// ds_i = [i kept] Gsum_i - g_i sum_{k kept} Gsum_k. The other activations of
// the method's comparison are listed at the terms below. One warp per
// (b, kv head, t) row; every column of the row is written.
__global__ void __launch_bounds__(256)
dscore_kernel(Shape sh, const float* __restrict__ scores, const float* __restrict__ slse,
              const int32_t* __restrict__ idx, const int32_t* __restrict__ nsel,
              const float* __restrict__ gsum, float* __restrict__ ds, const int* __restrict__ aborted) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= sh.rows()) return;
    if (aborted != nullptr && *aborted) {   // Gsum is incomplete: mark the row invalid
        for (int i = lane; i < sh.NB; i += 32) ds[row * sh.NB + i] = __int_as_float(0x7fc00000);
        return;
    }
    const bool r32 = sh.rows() <= (int64_t)UINT32_MAX;
    const int t = r32 ? (int)((uint32_t)row % (uint32_t)sh.T) : (int)(row % sh.T);
    const int C = r32 ? (int)(((uint32_t)sh.q_offset + (uint32_t)t) / (uint32_t)sh.bs)
                      : (int)(((int64_t)sh.q_offset + t) / sh.bs);
    const int mode = sh.gate;
    // every candidate gets -g_i * T (softmax gate and its straight-through
    // hard form), each kept block its own term on top
    const bool dense_term = mode == SAS_GATE_SOFTMAX || mode == SAS_GATE_STE;
    const float* sr = scores + row * sh.NB;
    float* dr = ds + row * sh.NB;
    // every load of the row is issued before any is used: the kept list, its
    // Gsum and scores (masked by n afterwards), the normaliser and the first
    // kPre chunks of 32 causal scores
    constexpr int kPre = 16;
    const int n = nsel[row];
    const float lse = slse[row];
    int si[2];
    float sg[2], sk[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int slot = lane + 32 * r;
        si[r] = slot < sh.K ? idx[row * sh.K + slot] : -1;
        sg[r] = slot < sh.K ? gsum[row * sh.K + slot] : 0.f;
    }
    float sv[kPre];
#pragma unroll
    for (int q = 0; q < kPre; ++q) {
        const int i = q * 32 + lane;
        sv[q] = (dense_term && i < C) ? sr[i] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (lane + 32 * r >= n || (unsigned)si[r] >= (unsigned)C) { si[r] = -1; sg[r] = 0.f; }
        sk[r] = si[r] >= 0 ? sr[si[r]] : -INFINITY;
    }
    float kv[2], T;
    dscore_kept_terms(mode, si, sg, sk, lse, kv, T);
    const bool any = mode != SAS_GATE_NONE;
    int base = 0;
    auto chunk = [&](int c0, float sc) {
        uint32_t bits = 0;
#pragma unroll
        for (int r = 0; r < 2; ++r)
            if (si[r] >= c0 && si[r] < c0 + 32) bits |= 1u << (si[r] - c0);
        const uint32_t mask = __reduce_or_sync(0xffffffffu, bits);
        const int slot = base + __popc(mask & ((1u << lane) - 1u));
        const float k0 = __shfl_sync(0xffffffffu, kv[0], slot & 31);
        const float k1 = __shfl_sync(0xffffffffu, kv[1], slot & 31);
        const int i = c0 + lane;
        float val = 0.f;
        if (any && i < C) {
            if (dense_term) val = -expf(sc - lse) * T;
            if ((mask >> lane) & 1u) val += slot < 32 ? k0 : k1;
        }
        if (i < sh.NB) dr[i] = val;
        base += __popc(mask);
    };
#pragma unroll
    for (int q = 0; q < kPre; ++q) {
        const int c0 = q * 32;
        if (c0 >= sh.NB) break;                        // warp-uniform
        chunk(c0, sv[q]);
    }
    for (int c0 = kPre * 32; c0 < sh.NB; c0 += 32)     // long rows: the rest one chunk at a time
        chunk(c0, (dense_term && c0 + lane < C) ? sr[c0 + lane] : 0.f);
}

// The same for rows of NB <= 128 * kPieces columns, NB % 4 == 0: lane l owns
// columns 4l .. 4l + 3 of each 128-column piece (16-byte loads and stores;
// kPieces 4 for rows of up to 512 columns, 8 up to 1024, so that the
// prefetched pieces hold no more registers than the row needs). Every
// column first gets its dense term (0 past C); after a warp barrier, which
// orders the warp's global stores, each kept slot's lane rewrites its column
// with the dense term plus its own term, computed as the scalar kernel does.
constexpr int kDsVecCols = 1024;
template <int kPieces>
__global__ void __launch_bounds__(256)
dscore_vec_kernel(Shape sh, const float* __restrict__ scores, const float* __restrict__ slse,
                  const int32_t* __restrict__ idx, const int32_t* __restrict__ nsel,
                  const float* __restrict__ gsum, float* __restrict__ ds, const int* __restrict__ aborted) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= sh.rows()) return;
    float4* dr = reinterpret_cast<float4*>(ds + row * sh.NB);
    const int nb4 = sh.NB / 4;
    if (aborted != nullptr && *aborted) {   // Gsum is incomplete: mark the row invalid
        const float nan = __int_as_float(0x7fc00000);
        for (int i = lane; i < nb4; i += 32) dr[i] = make_float4(nan, nan, nan, nan);
        return;
    }
    const bool r32 = sh.rows() <= (int64_t)UINT32_MAX;
    const int t = r32 ? (int)((uint32_t)row % (uint32_t)sh.T) : (int)(row % sh.T);
    const int C = r32 ? (int)(((uint32_t)sh.q_offset + (uint32_t)t) / (uint32_t)sh.bs)
                      : (int)(((int64_t)sh.q_offset + t) / sh.bs);
    const int mode = sh.gate;
    const bool dense_term = mode == SAS_GATE_SOFTMAX || mode == SAS_GATE_STE;
    const bool any = mode != SAS_GATE_NONE;
    const float* sr = scores + row * sh.NB;
    const float4* sr4 = reinterpret_cast<const float4*>(sr);
    const int n = nsel[row];
    const float lse = slse[row];
    int si[2];
    float sg[2], sk[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int slot = lane + 32 * r;
        si[r] = slot < sh.K ? idx[row * sh.K + slot] : -1;
        sg[r] = slot < sh.K ? gsum[row * sh.K + slot] : 0.f;
    }
    float4 sv[kPieces];
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
        const int i = q * 128 + 4 * lane;
        sv[q] = (dense_term && i < C) ? sr4[i / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (lane + 32 * r >= n || (unsigned)si[r] >= (unsigned)C) { si[r] = -1; sg[r] = 0.f; }
        sk[r] = si[r] >= 0 ? sr[si[r]] : -INFINITY;
    }
    float kv[2], T;
    dscore_kept_terms(mode, si, sg, sk, lse, kv, T);
    auto dense = [&](int i, float sc) { return (dense_term && i < C) ? -expf(sc - lse) * T : 0.f; };
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
        const int i = q * 128 + 4 * lane;
        if (i < sh.NB)
            dr[i / 4] = make_float4(dense(i, sv[q].x), dense(i + 1, sv[q].y), dense(i + 2, sv[q].z),
                                    dense(i + 3, sv[q].w));
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 2; ++r)
        if (any && si[r] >= 0) ds[row * sh.NB + si[r]] = dense(si[r], sk[r]) + kv[r];
}

template <typename T, int D, int GMAX, int BS>
cudaError_t run_fwd(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                    const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    const int64_t grid = (s.rows() + 3) / 4;
    KernelTimer kt("fwd_simt", st);
    fwd_simt_kernel<T, D, GMAX, BS><<<(unsigned)grid, 128, 0, st>>>(
        s, (const T*)q, (const T*)k, (const T*)v, idx, gl, nsel, (T*)o, lse, nullptr, nullptr);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

template <typename T, int D, int GMAX, int BS>
cudaError_t run_bwd(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                    const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                    const int32_t* nsel, const uint64_t* maskT, float* dq_acc, void* dk, void* dv,
                    float* dk32, float* dv32, float* gsum, cudaStream_t st) {
    constexpr int NT = BS * 4;
    const size_t smem = sizeof(float) * (2 * BS * (D + 4) + 2 * GMAX * D + GMAX * BS + 2 * GMAX + NT / 32);
    auto kern = bwd_simt_kernel<T, D, GMAX, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)s.B * s.Hkv * s.nT;
    {
        KernelTimer kt("bwd_simt", st);
        kern<<<(unsigned)grid, NT, smem, st>>>(s, (const T*)q, (const T*)k, (const T*)v, (const T*)dO, lse, Dd, idx,
                                               gl, nsel, maskT, dq_acc, (T*)dk, (T*)dv, dk32, dv32, gsum);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

template <typename T, int D, int BS>
cudaError_t fwd_g(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                  const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    if (s.G <= 4) return run_fwd<T, D, 4, BS>(s, q, k, v, idx, gl, nsel, o, lse, st);
    return run_fwd<T, D, 8, BS>(s, q, k, v, idx, gl, nsel, o, lse, st);
}
template <typename T, int D>
cudaError_t fwd_b(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                  const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    if (s.bs == 32) return fwd_g<T, D, 32>(s, q, k, v, idx, gl, nsel, o, lse, st);
    return fwd_g<T, D, 64>(s, q, k, v, idx, gl, nsel, o, lse, st);
}
template <typename T>
cudaError_t fwd_d(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                  const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    if (s.D == 64) return fwd_b<T, 64>(s, q, k, v, idx, gl, nsel, o, lse, st);
    return fwd_b<T, 128>(s, q, k, v, idx, gl, nsel, o, lse, st);
}

template <typename T, int D, int BS>
cudaError_t bwd_g(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                  const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                  const int32_t* nsel, const uint64_t* maskT, float* dq_acc, void* dk, void* dv,
                  float* dk32, float* dv32, float* gsum, cudaStream_t st) {
    if (s.G <= 4) return run_bwd<T, D, 4, BS>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
    return run_bwd<T, D, 8, BS>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
}
template <typename T, int D>
cudaError_t bwd_b(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                  const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                  const int32_t* nsel, const uint64_t* maskT, float* dq_acc, void* dk, void* dv,
                  float* dk32, float* dv32, float* gsum, cudaStream_t st) {
    if (s.bs == 32) return bwd_g<T, D, 32>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
    return bwd_g<T, D, 64>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
}
template <typename T>
cudaError_t bwd_d(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                  const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                  const int32_t* nsel, const uint64_t* maskT, float* dq_acc, void* dk, void* dv,
                  float* dk32, float* dv32, float* gsum, cudaStream_t st) {
    if (s.D == 64) return bwd_b<T, 64>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
    return bwd_b<T, 128>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
}

}  // namespace

cudaError_t launch_fwd_simt(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                            const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    if (s.dtype == SAS_DT_FP32) return fwd_d<float>(s, q, k, v, idx, gl, nsel, o, lse, st);
    return fwd_d<__nv_bfloat16>(s, q, k, v, idx, gl, nsel, o, lse, st);
}

cudaError_t launch_fwd_simt_rows(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                 const float* gl, const int32_t* nsel, const int32_t* list, const int32_t* list_n,
                                 void* o, float* lse, cudaStream_t st) {
    if (s.dtype != SAS_DT_BF16 || s.D != 128 || s.bs != 64) return cudaErrorInvalidValue;
    using B16 = __nv_bfloat16;
    const unsigned grid = 148;   // a few warps per SM; the rows to redo are normally none
    KernelTimer kt("fwd_rows_fixup", st);
    if (s.G <= 4)
        fwd_simt_kernel<B16, 128, 4, 64><<<grid, 128, 0, st>>>(s, (const B16*)q, (const B16*)k, (const B16*)v, idx, gl,
                                                               nsel, (B16*)o, lse, list, list_n);
    else
        fwd_simt_kernel<B16, 128, 8, 64><<<grid, 128, 0, st>>>(s, (const B16*)q, (const B16*)k, (const B16*)v, idx, gl,
                                                               nsel, (B16*)o, lse, list, list_n);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t launch_bwd_rowdot(const Shape& s, const void* o, const void* dO, float* Dd, float* dq_acc,
                              cudaStream_t st) {
    const int64_t rows = (int64_t)s.B * s.Hq * s.T;
    // 8 warps per CTA, at least 8 rows per warp pass; at most 16 CTAs per SM
    const unsigned grid = (unsigned)std::min<int64_t>((rows + 63) / 64, 148 * 16);
    KernelTimer kt("rowdot", st);
    if (s.dtype == SAS_DT_FP32) {
        if (s.D == 64) rowdot_kernel<float, 64><<<grid, 256, 0, st>>>(rows, (const float*)o, (const float*)dO, Dd,
                                                                    dq_acc);
        else rowdot_kernel<float, 128><<<grid, 256, 0, st>>>(rows, (const float*)o, (const float*)dO, Dd,
                                                                    dq_acc);
    } else {
        using B16 = __nv_bfloat16;
        if (s.D == 64) rowdot_kernel<B16, 64><<<grid, 256, 0, st>>>(rows, (const B16*)o, (const B16*)dO, Dd,
                                                                    dq_acc);
        else rowdot_kernel<B16, 128><<<grid, 256, 0, st>>>(rows, (const B16*)o, (const B16*)dO, Dd,
                                                                    dq_acc);
    }
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t launch_bwd_simt(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                            const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                            const int32_t* nsel, const uint64_t* maskT, float* dq_acc, void* dk, void* dv,
                            float* dk32, float* dv32, float* gsum, cudaStream_t st) {
    if (s.dtype == SAS_DT_FP32)
        return bwd_d<float>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
    return bwd_d<__nv_bfloat16>(s, q, k, v, dO, lse, Dd, idx, gl, nsel, maskT, dq_acc, dk, dv, dk32, dv32, gsum, st);
}

cudaError_t launch_cast_dq(const Shape& s, const float* dq_acc, void* dq, const int* aborted, cudaStream_t st) {
    // bf16 only: fp32 accumulates dq in place. n is a multiple of 8 (d is 64 or
    // 128); both buffers are 16-byte aligned.
    if (s.dtype != SAS_DT_BF16) return cudaErrorInvalidValue;
    const int64_t n8 = (int64_t)s.B * s.Hq * s.T * s.D / 8;
    const unsigned g8 = (unsigned)std::min<int64_t>((n8 + 511) / 512, 148 * 8);
    {
        KernelTimer kt("cast_dq", st);
        cast_bf16x8_kernel<<<g8, 256, 0, st>>>(n8, reinterpret_cast<const float4*>(dq_acc), static_cast<uint4*>(dq),
                                               aborted);
    }
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t launch_dscore(const Shape& s, const float* scores, const float* slse, const int32_t* idx,
                          const int32_t* nsel, const float* gsum, float* ds, const int* aborted, cudaStream_t st) {
    const unsigned grid = (unsigned)((s.rows() + 7) / 8);
    KernelTimer kt("dscore", st);
    const bool vec = s.NB % 4 == 0 && s.NB <= kDsVecCols && ((uintptr_t)scores & 15) == 0 && ((uintptr_t)ds & 15) == 0;
    if (vec && s.NB <= 512)
        dscore_vec_kernel<4><<<grid, 256, 0, st>>>(s, scores, slse, idx, nsel, gsum, ds, aborted);
    else if (vec)
        dscore_vec_kernel<8><<<grid, 256, 0, st>>>(s, scores, slse, idx, nsel, gsum, ds, aborted);
    else
        dscore_kernel<<<grid, 256, 0, st>>>(s, scores, slse, idx, nsel, gsum, ds, aborted);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas

namespace sas {

cudaError_t launch_reduce_dkv(const Shape& s, const float* dk32, const float* dv32, void* dk, void* dv,
                              cudaStream_t st) {
    const int64_t n = (int64_t)s.B * s.Hkvp * s.T * s.D / 4;
    const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 8);
    KernelTimer kt("reduce_dkv", st);
    if (s.dtype == SAS_DT_FP32)
        reduce_dkv_kernel<float><<<grid, 256, 0, st>>>(s, dk32, dv32, (float*)dk, (float*)dv);
    else
        reduce_dkv_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(s, dk32, dv32, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace sas
