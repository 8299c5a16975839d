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

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

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

// ---------------------------------------------------------------------------
// Tensor-core variant (bf16, d = 128, block 64, G <= 8). Warp 0 moves blocks
// into a 4-stage ring by TMA (K and V as two 64-column boxes each, 128-byte
// swizzle); warps 1 and 2 each own every other stage and run the whole block
// on mma.sync m16n8k16 with no CTA-wide barrier:
//   S^T = K q^T   (M = 16 keys, N = 8 heads, K = 16 dims; 4 x 8 MMAs)
//   online softmax per head in log2 units (scale applied in fp32 after the MMA)
//   O^T += V^T P^T (M = 16 dims, N = 8 heads, K = 16 keys; 8 x 4 MMAs)
// K rows come through ldmatrix, V rows through ldmatrix.trans, and the P tile
// (keys x heads, accumulator layout) becomes the B operand by movmatrix.trans.
// Rows of the current block at or after the new token may hold anything in the
// cache: their scores are replaced by -inf and their V rows zeroed in shared
// memory before the product. The two consumers merge their (m, l, O) at the
// end and write one partial per CTA for the same merge kernel.
constexpr int kMmaStages = 4;
constexpr uint32_t kMmaStage = 32768;   // K box 0 | K box 1 | V box 0 | V box 1, 8 KiB each

struct DecMmaArgs {
    DecArgs d;
};

__device__ __forceinline__ uint32_t sw_addr(uint32_t box, int row, int chunk) {
    return box + (uint32_t)row * 128u + (uint32_t)((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(96, 1)
decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ DecMmaArgs args) {
    constexpr int D = 128, BS = 64;
    const DecArgs& a = args.d;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kMmaStages * kMmaStage);
    uint64_t* empty = full + kMmaStages;
    float* xch = reinterpret_cast<float*>(empty + kMmaStages);   // consumer 1's m[8], l[8], O^T[128][8]

    const Shape& sh = a.sh;
    const int G = sh.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x % a.splits;
    const int64_t bg = blockIdx.x / a.splits;
    const int b = (int)(bg / sh.Hkv), g = (int)(bg % sh.Hkv);
    const int64_t N = (int64_t)sh.q_offset + 1;
    const int C = (int)(sh.q_offset / BS);
    const bool dense = a.idx == nullptr;
    const int n = dense ? C : a.nsel[bg];
    const int nblk = n + 1;
    const int p0 = split * a.bpc;
    const int cnt = max(min(p0 + a.bpc, nblk) - p0, 0);
    auto block_of = [&](int pos) -> int {
        if (dense) return pos;
        if (pos >= n) return C;
        const int j = a.idx[bg * sh.K + pos];
        return ((unsigned)j < (unsigned)C) ? j : -1;
    };
    auto ntok_of = [&](int j) -> int { return j < 0 ? 0 : (j == C ? (int)(N - (int64_t)C * BS) : BS); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMmaStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---- producer ----
        if (lane == 0) {
            for (int i = 0; i < cnt; ++i) {
                const int s = i % kMmaStages;
                if (i >= kMmaStages && !mbar_wait_bounded(&empty[s], (uint32_t)(((i / kMmaStages) - 1) & 1))) break;
                const int j = block_of(p0 + i);
                if (j < 0) {
                    tc::mbar_arrive(&full[s]);
                    continue;
                }
                mbar_arrive_expect_tx(&full[s], kMmaStage);
                const int row = (int)(bg * a.stride + (int64_t)j * BS);
                unsigned char* st = sm + s * kMmaStage;
                tc::tma_load_2d(st, &tm_k, 0, row, &full[s]);
                tc::tma_load_2d(st + 8192, &tm_k, 64, row, &full[s]);
                tc::tma_load_2d(st + 16384, &tm_v, 0, row, &full[s]);
                tc::tma_load_2d(st + 24576, &tm_v, 64, row, &full[s]);
            }
        }
        return;
    }

    // ---- consumers: warp 1 takes blocks 0, 2, ...; warp 2 blocks 1, 3, ... ----
    const int cw = warp - 1;
    const int gq = lane >> 2, tq = lane & 3;
    const float qk = sh.scale * kLog2e;
    // q^T as the B operand: b0 = q[head gq][16 ks + 2 tq, +1], b1 = the same + 8
    uint32_t qb[8][2];
    {
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + ((int64_t)b * sh.Hq + (int64_t)g * G) * D;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            if (gq < G) {
                qb[ks][0] = *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * ks + 2 * tq);
                qb[ks][1] = *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * ks + 2 * tq + 8);
            } else {
                qb[ks][0] = qb[ks][1] = 0u;
            }
        }
    }
    float o[8][4];          // O^T: m-tile of 16 dims, (dim gq | gq+8) x (heads 2tq, 2tq+1)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
    float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};   // heads 2tq, 2tq+1

    const uint32_t sbase = smem_u32(sm);
    bool ok = true;
    for (int i = cw; i < cnt; i += 2) {
        const int s = i % kMmaStages;
        if (!mbar_wait_bounded(&full[s], (uint32_t)((i / kMmaStages) & 1))) { ok = false; break; }
        const int j = block_of(p0 + i);
        const int ntok = ntok_of(j);
        if (ntok > 0) {
            const uint32_t kb0 = sbase + s * kMmaStage, kb1 = kb0 + 8192, vb0 = kb0 + 16384, vb1 = kb0 + 24576;
            if (ntok < BS) {   // the current block: clear V rows >= ntok (128 bytes per row and box)
                unsigned char* v0p = sm + s * kMmaStage + 16384;
                for (int e = ntok * 8 + lane; e < BS * 8; e += 32) {
                    reinterpret_cast<uint4*>(v0p)[e] = make_uint4(0, 0, 0, 0);
                    reinterpret_cast<uint4*>(v0p + 8192)[e] = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            const float lg = (!dense && p0 + i < n) ? a.gl[bg * sh.K + p0 + i] * kLog2e : 0.f;
            // ---- S^T = K q^T ----
            float sc[4][4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    // matrices: (keys +0..7, dims +0..7), (keys +8..15, dims +0..7), (keys +0..7, dims +8..15), (keys +8.., dims +8..)
                    const int key = 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int chunk = 2 * ks + (lane >> 4);
                    const uint32_t addr = sw_addr(chunk < 8 ? kb0 : kb1, key, chunk & 7);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(addr, a0, a1, a2, a3);
                    mma_bf16(sc[mt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                }
            }
            // ---- online softmax (heads 2tq, 2tq+1; keys 16 mt + gq (+8)) ----
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = 16 * mt + gq + (e >> 1) * 8;
                    const float v = key < ntok ? fmaf(sc[mt][e], qk, lg) : -INFINITY;
                    sc[mt][e] = v;
                    mx[e & 1] = fmaxf(mx[e & 1], v);
                }
            float corr[2], psum[2] = {0.f, 0.f};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
                const float mn = fmaxf(mrun[h], mx[h]);
                corr[h] = mrun[h] == -INFINITY ? 0.f : exp2f(mrun[h] - mn);
                mrun[h] = mn;
            }
            uint32_t pb[4][2];   // P^T as B operand per k-step (16 keys)
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m = mrun[e & 1];
                    p[e] = m == -INFINITY ? 0.f : exp2f(sc[mt][e] - m);
                    psum[e & 1] += p[e];
                }
                pb[mt][0] = movm_t(pack_bf16(p[0], p[1]));   // keys 16 mt + 0..7
                pb[mt][1] = movm_t(pack_bf16(p[2], p[3]));   // keys 16 mt + 8..15
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 4);
                psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 8);
                psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 16);
                lrun[h] = lrun[h] * corr[h] + psum[h];
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                o[mt][0] *= corr[0];
                o[mt][1] *= corr[1];
                o[mt][2] *= corr[0];
                o[mt][3] *= corr[1];
            }
            // ---- O^T += V^T P^T ----
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {        // dims 16 mt .. + 15
#pragma unroll
                for (int kst = 0; kst < 4; ++kst) { // keys 16 kst .. + 15
                    // matrices (transposed on load): (keys +0..7, dims +0..7), (keys +0..7, dims +8..15),
                    // (keys +8..15, dims +0..7), (keys +8..15, dims +8..15)
                    const int key = 16 * kst + (lane & 7) + (lane >> 4) * 8;
                    const int chunk = 2 * mt + ((lane >> 3) & 1);
                    const uint32_t addr = sw_addr(chunk < 8 ? vb0 : vb1, key, chunk & 7);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(addr, a0, a1, a2, a3);
                    mma_bf16(o[mt], a0, a1, a2, a3, pb[kst][0], pb[kst][1]);
                }
            }
        }
        tc::fence_async_shared();   // the zeroed rows are rewritten by TMA next
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[s]);
    }

    // ---- merge the two consumers; consumer 0 writes the CTA's partial ----
    float* rec = a.part + (bg * a.splits + split) * (int64_t)G * (D + 2);
    if (cw == 1) {
        if (gq == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) { xch[2 * tq + h] = mrun[h]; xch[8 + 2 * tq + h] = lrun[h]; }
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int dim = 16 * mt + gq + (e >> 1) * 8, h = 2 * tq + (e & 1);
                xch[16 + dim * 8 + h] = o[mt][e];
            }
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    if (cw == 0) {
        float m2[2], l2[2], w1[2], w2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            m2[h] = xch[2 * tq + h];
            l2[h] = xch[8 + 2 * tq + h];
            const float M = fmaxf(mrun[h], m2[h]);
            w1[h] = mrun[h] == -INFINITY ? 0.f : exp2f(mrun[h] - M);
            w2[h] = m2[h] == -INFINITY ? 0.f : exp2f(m2[h] - M);
            mrun[h] = M;
            lrun[h] = lrun[h] * w1[h] + l2[h] * w2[h];
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int dim = 16 * mt + gq + (e >> 1) * 8, h = 2 * tq + (e & 1);
                const float v = o[mt][e] * w1[e & 1] + xch[16 + dim * 8 + h] * w2[e & 1];
                if (h < G) rec[h * (D + 2) + dim] = ok ? v : __int_as_float(0x7fc00000);
            }
        if (gq == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int hh = 2 * tq + h;
                if (hh < G) {
                    rec[hh * (D + 2) + D] = mrun[h];
                    rec[hh * (D + 2) + D + 1] = lrun[h];
                }
            }
        }
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

cudaError_t run_decode_mma(const DecArgs& a, cudaStream_t st) {
    CUtensorMap mk, mv;
    const uint64_t rows = (uint64_t)a.sh.B * a.sh.Hkv * (uint64_t)a.stride;
    if (!encode_bf16_2d(&mk, a.kc, rows, 128, 64) || !encode_bf16_2d(&mv, a.vc, rows, 128, 64))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)kMmaStages * kMmaStage + 2 * kMmaStages * 8 + sizeof(float) * (16 + 128 * 8) + 1024;
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)a.sh.B * a.sh.Hkv * a.splits;
    {
        KernelTimer kt("decode_partial", st);
        decode_mma_kernel<<<(unsigned)grid, 96, smem, st>>>(mk, mv, DecMmaArgs{a});
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    {
        KernelTimer kt("decode_combine", st);
        decode_combine_kernel<__nv_bfloat16, 128><<<(unsigned)(a.sh.B * a.sh.Hkv * a.sh.G), 128, 0, st>>>(
            a.sh, a.part, a.splits, static_cast<__nv_bfloat16*>(a.o));
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

static bool decode_mma_supported(const Shape& s) {
    return s.dtype == SAS_DT_BF16 && s.D == 128 && s.bs == 64 && s.G <= 8;
}

DecodePlan decode_plan(const Shape& s, bool dense) {
    DecodePlan p;
    const int64_t C = s.q_offset / s.bs;
    if (decode_mma_supported(s)) {
        // one CTA per SM (128 KiB of stages); two blocks per CTA for a
        // selection, one wave of CTAs over every block for dense
        const int64_t nblk = dense ? C + 1 : (int64_t)s.K + 1;
        const int64_t groups = (int64_t)s.B * s.Hkv;
        int64_t bpc = dense ? (groups * nblk + 147) / 148 : 2;
        bpc = std::max<int64_t>(bpc, (nblk + kMaxSplits - 1) / kMaxSplits);
        bpc = std::max<int64_t>(1, bpc);
        p.bpc = (int)bpc;
        p.splits = (int)((nblk + bpc - 1) / bpc);
        return p;
    }
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
    if (decode_mma_supported(s)) return run_decode_mma(a, st);
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
