// decode.cu -- budgeted sparse decode (and dense decode) over a KV cache.
//
// One new token per (batch, query head) at position N - 1 attends the K kept
// historical blocks of its KV group plus the causal current block
// (SAS study note 3-7 inference path, steps 2-4). With no selection it attends
// every token [0, N) with no gate: the dense comparison of study note 5-6.
//
// Work split: the block list of each (b, kv head) is cut into `splits` chunks
// of `bpc` blocks; one CTA per chunk streams its blocks through two shared
// memory stages. Each block's K and V rows are contiguous in the cache, so one
// bulk async copy per tensor moves a whole block (16 KiB at b=64, d=128, bf16)
// with a single instruction. The CTA writes an unnormalised partial (m, l, o)
// for the G heads, and a second kernel merges the partials by log-sum-exp.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {

constexpr int kDecThreads = 256;

struct DecArgs {
    Shape sh;
    const void* q;
    const void* kc;
    const void* vc;
    int64_t stride;      // cache tokens per (b, kv head)
    const int32_t* idx;  // nullptr: dense
    const float* gl;
    const int32_t* nsel;
    float* part;         // [B*Hkv][splits][G][D + 2]: o (unnormalised), m (log2 units), l
    void* o;             // [B, Hq, D] output
    int bpc;
    int splits;
};

template <typename T, int D, int BS>
constexpr size_t dec_stage_bytes() { return (size_t)2 * BS * D * sizeof(T); }

// Region 0 holds the two stages while streaming and the cross-key-group
// reduction buffer [NKG][GMAX][D] afterwards.
template <typename T, int D, int GMAX, int BS>
constexpr size_t dec_region0_bytes() {
    constexpr size_t stages = 2 * dec_stage_bytes<T, D, BS>();
    constexpr size_t red = (size_t)(kDecThreads / (D * (int)sizeof(T) / 16)) * GMAX * D * sizeof(float);
    return stages > red ? stages : red;
}

template <typename T, int D, int GMAX, int BS>
constexpr size_t dec_smem_bytes() {
    // region 0; q [GMAX][D]; p [BS][GMAX]; m,l,corr [GMAX]; 2 mbarriers; flag.
    return dec_region0_bytes<T, D, GMAX, BS>() + sizeof(float) * (GMAX * D + BS * GMAX + 3 * GMAX + 1) + 2 * 8 +
           16;
}

template <typename T, int D, int GMAX, int BS>
__global__ void __launch_bounds__(kDecThreads)
decode_partial_kernel(DecArgs a) {
    constexpr int VE = vec16<T>();             // elements per 16-byte chunk
    constexpr int CPR = D * (int)sizeof(T) / 16;  // chunks per row
    constexpr int NKG = kDecThreads / CPR;     // key groups in the PV phase
    constexpr int CPT = CPR / 8;               // chunks per thread in the score phase
    constexpr size_t STAGE = dec_stage_bytes<T, D, BS>();
    constexpr size_t HALF = STAGE / 2;
    static_assert(CPR % 8 == 0 && kDecThreads % CPR == 0, "layout");

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* stage_base = smem;
    constexpr size_t R0 = dec_region0_bytes<T, D, GMAX, BS>();
    float* qs = reinterpret_cast<float*>(smem + R0);          // [GMAX][D], pre-scaled to log2 units
    float* ps = qs + GMAX * D;                                 // [BS][GMAX]
    float* st_m = ps + BS * GMAX;
    float* st_l = st_m + GMAX;
    float* st_c = st_l + GMAX;
    uint64_t* bars = reinterpret_cast<uint64_t*>(st_c + GMAX + (GMAX & 1));
    int* flag = reinterpret_cast<int*>(bars + 2);

    const Shape& sh = a.sh;
    const int G = sh.G;
    const int tid = threadIdx.x;
    const int split = blockIdx.x % a.splits;
    const int64_t bg = blockIdx.x / a.splits;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int64_t N = (int64_t)sh.q_offset + 1;
    const int C = (int)(sh.q_offset / BS);
    const bool dense = a.idx == nullptr;
    const int n = dense ? C : a.nsel[bg];
    const int nblk = n + 1;
    const int p0 = split * a.bpc;
    const int p1 = min(p0 + a.bpc, nblk);
    const int cnt = max(p1 - p0, 0);

    const T* kc = static_cast<const T*>(a.kc) + bg * a.stride * D;
    const T* vc = static_cast<const T*>(a.vc) + bg * a.stride * D;

    // An index outside [0, C) is not a valid selection: such a block is
    // skipped (no copy, no keys) rather than read out of bounds.
    auto block_of = [&](int pos) -> int {
        if (dense) return pos;
        if (pos >= n) return C;
        const int j = a.idx[bg * sh.K + pos];
        return ((unsigned)j < (unsigned)C) ? j : -1;
    };
    auto ntok_of = [&](int j) -> int { return j < 0 ? 0 : (j == C ? (int)(N - (int64_t)C * BS) : BS); };
    auto issue = [&](int i) {  // thread 0 only: block p0 + i into stage i & 1
        const int j = block_of(p0 + i);
        const uint32_t bytes = (uint32_t)ntok_of(j) * D * (uint32_t)sizeof(T);
        unsigned char* dst = stage_base + (size_t)(i & 1) * STAGE;
        mbar_arrive_expect_tx(&bars[i & 1], 2 * bytes);
        if (bytes > 0) {
            bulk_g2s(dst, kc + (int64_t)j * BS * D, bytes, &bars[i & 1]);
            bulk_g2s(dst + HALF, vc + (int64_t)j * BS * D, bytes, &bars[i & 1]);
        }
    };

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < cnt && i < 2; ++i) issue(i);
    }
    const float qscale = sh.scale * kLog2e;
    const T* qg = static_cast<const T*>(a.q) + ((int64_t)b * sh.Hq + (int64_t)g * G) * D;
    for (int e = tid; e < GMAX * D; e += kDecThreads) qs[e] = e < G * D ? Elem<T>::to_f(qg[e]) * qscale : 0.f;
    if (tid < GMAX) { st_m[tid] = -INFINITY; st_l[tid] = 0.f; st_c[tid] = 1.f; }

    // PV-phase ownership: chunk c (VE dims) of keys kg, kg + NKG, ...
    const int pc = tid % CPR, kg = tid / CPR;
    float acc[GMAX][VE];
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[h][e] = 0.f;
    // score-phase ownership: key sk = tid / 8 (+32 per round), chunks c8 + 8i
    const int c8 = tid & 7;

    int failed = -1;
    for (int i = 0; i < cnt; ++i) {
        const int j = block_of(p0 + i);
        const int ntok = ntok_of(j);
        const float lg = (!dense && p0 + i < n) ? a.gl[bg * sh.K + p0 + i] * kLog2e : 0.f;
        if (tid == 0) flag[0] = mbar_wait_bounded(&bars[i & 1], (uint32_t)((i >> 1) & 1)) ? 1 : 0;
        __syncthreads();
        if (!flag[0]) { failed = i; break; }
        const T* Ks = reinterpret_cast<const T*>(stage_base + (size_t)(i & 1) * STAGE);
        const T* Vs = reinterpret_cast<const T*>(stage_base + (size_t)(i & 1) * STAGE + HALF);

        // ---- scores: 8 threads per key, reduced by shuffles ----
#pragma unroll
        for (int r = 0; r < BS / 32; ++r) {
            const int sk = (tid >> 3) + 32 * r;
            float s[GMAX];
#pragma unroll
            for (int h = 0; h < GMAX; ++h) s[h] = 0.f;
            if (sk < ntok) {
#pragma unroll
                for (int ci = 0; ci < CPT; ++ci) {
                    const int c = c8 + 8 * ci;
                    float kv[VE];
                    load_vec<T, VE>(Ks + sk * D + c * VE, kv);
#pragma unroll
                    for (int h = 0; h < GMAX; ++h) {
                        if (h < G) {
#pragma unroll
                            for (int e = 0; e < VE; ++e) s[h] = fmaf(qs[h * D + c * VE + e], kv[e], s[h]);
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 1);
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 2);
                s[h] += __shfl_xor_sync(0xffffffffu, s[h], 4);
            }
            if (c8 == 0 && sk < BS) {
#pragma unroll
                for (int h = 0; h < GMAX; ++h) ps[sk * GMAX + h] = sk < ntok ? s[h] + lg : -INFINITY;
            }
        }
        __syncthreads();

        // ---- online softmax: warp h owns head h ----
        {
            const int w = tid >> 5, lane = tid & 31;
            if (w < G) {
                float x[BS / 32];
                float mx = -INFINITY;
#pragma unroll
                for (int r = 0; r < BS / 32; ++r) { x[r] = ps[(lane + 32 * r) * GMAX + w]; mx = fmaxf(mx, x[r]); }
                mx = warp_max(mx);
                const float mo = st_m[w];
                const float mn = fmaxf(mo, mx);
                float sum = 0.f;
#pragma unroll
                for (int r = 0; r < BS / 32; ++r) {
                    const float pv = mn == -INFINITY ? 0.f : exp2f(x[r] - mn);
                    ps[(lane + 32 * r) * GMAX + w] = pv;
                    sum += pv;
                }
                sum = warp_sum(sum);
                if (lane == 0) {
                    const float corr = mo == -INFINITY ? 0.f : exp2f(mo - mn);
                    st_c[w] = corr;
                    st_l[w] = st_l[w] * corr + sum;
                    st_m[w] = mn;
                }
            }
        }
        __syncthreads();

        // ---- o = o * corr + P V ----
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            const float c = st_c[h];
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[h][e] *= c;
        }
        for (int key = kg; key < ntok; key += NKG) {
            float vv[VE];
            load_vec<T, VE>(Vs + key * D + pc * VE, vv);
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                const float pk = ps[key * GMAX + h];
#pragma unroll
                for (int e = 0; e < VE; ++e) acc[h][e] = fmaf(pk, vv[e], acc[h][e]);
            }
        }
        __syncthreads();   // every thread is done with this stage and with ps
        if (tid == 0 && i + 2 < cnt) issue(i + 2);
    }

    if (failed >= 0) {
        // A copy never completed: wait (bounded) for the copies still in
        // flight into this CTA's shared memory, then leave NaN partials so the
        // result is visibly invalid.
        if (tid == 0) {
            for (int i = failed; i < cnt && i < failed + 2; ++i)
                mbar_wait_bounded(&bars[i & 1], (uint32_t)((i >> 1) & 1));
        }
        __syncthreads();
        float* rec = a.part + (bg * a.splits + split) * (int64_t)G * (D + 2);
        for (int e = tid; e < G * (D + 2); e += kDecThreads) rec[e] = __int_as_float(0x7fc00000);
        return;
    }

    // ---- reduce acc over the NKG key groups (reusing the stage buffers) ----
    float* red = reinterpret_cast<float*>(stage_base);   // [NKG][GMAX][D], fits region 0
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
#pragma unroll
        for (int e = 0; e < VE; ++e) red[((size_t)kg * GMAX + h) * D + pc * VE + e] = acc[h][e];
    __syncthreads();
    float* rec = a.part + (bg * a.splits + split) * (int64_t)G * (D + 2);
    for (int e = tid; e < G * D; e += kDecThreads) {
        const int h = e / D, d = e % D;
        float s = 0.f;
#pragma unroll 4
        for (int x = 0; x < NKG; ++x) s += red[((size_t)x * GMAX + h) * D + d];
        rec[h * (D + 2) + d] = s;
    }
    if (tid < G) {
        rec[tid * (D + 2) + D] = st_m[tid];
        rec[tid * (D + 2) + D + 1] = st_l[tid];
    }
}

// Merge the splits of one (b, kv head, query head):
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
// The split weights are formed once in shared memory; each thread then reads
// its output column of every split with independent loads.
constexpr int kMaxSplits = 1024;

template <typename T, int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(Shape sh, const float* __restrict__ part, int splits, T* __restrict__ o) {
    __shared__ float w[kMaxSplits];
    __shared__ float red[4];
    const int G = sh.G;
    const int h = blockIdx.x % G;
    const int64_t bg = blockIdx.x / G;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    auto rec = [&](int s) { return part + ((bg * splits + s) * G + h) * (int64_t)(D + 2); };
    float m = -INFINITY;
    for (int s = tid; s < splits; s += 128) m = fmaxf(m, rec(s)[D]);
    m = warp_max(m);
    if (lane == 0) red[wp] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float l = 0.f;
    for (int s = tid; s < splits; s += 128) {
        const float* r = rec(s);
        const float ws = r[D] == -INFINITY ? 0.f : exp2f(r[D] - M);
        w[s] = ws;
        l = fmaf(ws, r[D + 1], l);
    }
    l = warp_sum(l);
    if (lane == 0) red[wp] = l;
    __syncthreads();
    const float L = red[0] + red[1] + red[2] + red[3];
    for (int d = tid; d < D; d += 128) {
        float acc = 0.f;
#pragma unroll 8
        for (int s = 0; s < splits; ++s) acc = fmaf(w[s], rec(s)[d], acc);
        o[((int64_t)b * sh.Hq + (int64_t)g * G + h) * D + d] = Elem<T>::from_f(acc / L);
    }
}

template <typename T, int D, int GMAX, int BS>
cudaError_t run_decode(const DecArgs& a, cudaStream_t st) {
    constexpr size_t smem = dec_smem_bytes<T, D, GMAX, BS>();
    auto kern = decode_partial_kernel<T, D, GMAX, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)a.sh.B * a.sh.Hkv * a.splits;
    {
        KernelTimer kt("decode_partial", st);
        kern<<<(unsigned)grid, kDecThreads, smem, st>>>(a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    {
        KernelTimer kt("decode_combine", st);
        decode_combine_kernel<T, D><<<(unsigned)(a.sh.B * a.sh.Hkv * a.sh.G), 128, 0, st>>>(a.sh, a.part, a.splits,
                                                                                           static_cast<T*>(a.o));
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

template <typename T, int D, int BS>
cudaError_t decode_g(const DecArgs& a, cudaStream_t st) {
    if (a.sh.G <= 4) return run_decode<T, D, 4, BS>(a, st);
    return run_decode<T, D, 8, BS>(a, st);
}
template <typename T, int D>
cudaError_t decode_b(const DecArgs& a, cudaStream_t st) {
    if (a.sh.bs == 32) return decode_g<T, D, 32>(a, st);
    return decode_g<T, D, 64>(a, st);
}
template <typename T>
cudaError_t decode_d(const DecArgs& a, cudaStream_t st) {
    if (a.sh.D == 64) return decode_b<T, 64>(a, st);
    return decode_b<T, 128>(a, st);
}

}  // namespace

DecodePlan decode_plan(const Shape& s, bool dense) {
    DecodePlan p;
    const int64_t C = s.q_offset / s.bs;
    if (!dense) {
        p.bpc = 1;
        p.splits = s.K + 1;
        return p;
    }
    const int64_t nblk = C + 1;
    const int64_t groups = (int64_t)s.B * s.Hkv;
    const int64_t target = 148 * 3;   // CTAs: one wave (three ~67 KB, 256-thread CTAs fit per SM)
    int64_t bpc = (groups * nblk + target - 1) / target;
    bpc = std::max<int64_t>(bpc, (nblk + kMaxSplits - 1) / kMaxSplits);   // the merge takes <= kMaxSplits
    bpc = std::max<int64_t>(1, bpc);
    p.bpc = (int)bpc;
    p.splits = (int)((nblk + bpc - 1) / bpc);
    return p;
}

cudaError_t launch_decode(const Shape& s, const void* q, const void* kc, const void* vc, int64_t stride,
                          const int32_t* idx, const float* gl, const int32_t* nsel, void* o, float* part,
                          cudaStream_t st) {
    const DecodePlan p = decode_plan(s, idx == nullptr);
    DecArgs a{s, q, kc, vc, stride, idx, gl, nsel, part, o, p.bpc, p.splits};
    if (s.dtype == SAS_DT_FP32) return decode_d<float>(a, st);
    return decode_d<__nv_bfloat16>(a, st);
}

cudaError_t read_decode_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

size_t decode_ws_bytes(const Shape& s) {
    const DecodePlan a = decode_plan(s, false), b = decode_plan(s, true);
    const int64_t splits = std::max(a.splits, b.splits);
    return sizeof(float) * (size_t)s.B * s.Hkv * splits * s.G * (s.D + 2);
}

}  // namespace sas

// ------------------------------------------------- decode without allocation ---
//
// Some callers of decode cannot call cudaMalloc at all: code that runs with a
// fixed memory budget carved out up front, plug-ins whose host framework owns
// every device allocation, or paths where an allocation (or its implicit
// synchronisation) is not allowed. For them, sas_sparse_decode_noalloc keeps the
// split partials in this file-scope device array instead of a caller workspace.
// Every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAS_NOALLOC_SCRATCH_BYTES];

namespace sas {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t noalloc_scratch(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<float*>(g_scratch_ptr[dev]);
    return cudaSuccess;
}

}  // namespace

}  // namespace sas

extern "C" sas_status sas_sparse_decode_noalloc(const sas_desc* desc, const void* q, const void* k_cache,
                                                const void* v_cache, int64_t cache_stride_tokens,
                                                const int32_t* idx, const float* gate_logit,
                                                const int32_t* n_sel, void* o, void* stream) {
    using namespace sas;
    Shape s;
    sas_status st = check_decode_args(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o, &s);
    if (st != SAS_OK) return st;
    const DecodePlan p = decode_plan(s, idx == nullptr);
    const size_t need = sizeof(float) * (size_t)s.B * s.Hkv * p.splits * s.G * (s.D + 2);
    if (need > (size_t)SAS_NOALLOC_SCRATCH_BYTES) return SAS_ERR_WORKSPACE;
    float* part = nullptr;
    if (noalloc_scratch(&part) != cudaSuccess) return SAS_ERR_CUDA;
    // Every split record is written before the merge reads it, so nothing in
    // the shared array has to start at zero.
    const cudaError_t e = launch_decode(s, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o,
                                        part, (cudaStream_t)stream);
    return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA;
}
