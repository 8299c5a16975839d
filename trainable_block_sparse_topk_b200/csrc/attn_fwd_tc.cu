// attn_fwd_tc.cu -- gated block-sparse forward on the sm_100a tensor cores.
//
// Computes, for every query row, o = softmax(a) V with
//   a_j = scale * q . k_j + log g_blk(j) on the tokens of the row's kept blocks,
//   a_j = scale * q . k_j                on the current block, j <= p
// (SAS study note 2-2 gated-attention eq.; arXiv text 4, inner log-space gate
// in FlashAttention-style tiles, study note 3-6).
//
// Tiling. One CTA owns a 64-token query tile tau (which is also the tokens'
// current block) of one KV group and two of its query heads: 128 rows, one
// tcgen05 M=128 tile. Because the G heads of a token share its selection, the
// CTA walks the union of its 64 tokens' kept blocks (ascending) and then the
// diagonal block tau; for each it computes S = Q K^T (M=128, N=64, K=d) into
// TMEM, the softmax warps turn S into P with the row's own mask (kept block ->
// + log gate, not kept -> masked out, diagonal -> causal), and the MMA adds
// P V into the TMEM accumulator O. Rows that did not keep a block contribute
// exact zeros, so the result equals the per-row definition.
//
// Roles (256 threads): warp 0 lane 0 issues TMA loads (Q once; K and V of each
// union block into a 3-stage ring), warp 1 lane 0 issues the MMAs, warp 2 owns
// the TMEM allocation, warps 4-7 run the softmax (thread = row = TMEM lane) and
// the epilogue. TMEM: S double buffer in columns [0,128), O in [128, 128+d).
// Softmax runs in log2 units with a lazily updated row maximum: O is rescaled
// only when a new maximum exceeds the one in use by more than 8 (P stays
// <= 2^8, exact in fp32 accumulation and bf16 range).
//
// All shared-memory operand tiles are 128-byte swizzled, 1024-byte aligned;
// K and Q are K-major operands, V is an MN-major operand of P V, P is written
// K-major by the softmax threads. No TMA multicast is used.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sas {

namespace {

constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kBS = 64;          // keys per block
constexpr int kTok = 64;         // query tokens per CTA
constexpr int kMaxNB = 1024;     // blocks per sequence handled by this kernel
constexpr uint32_t kTmemCols = 256;

struct FwdTcArgs {
    Shape sh;
    const int32_t* idx;
    const float* gl;
    const int32_t* nsel;
    __nv_bfloat16* o;
    float* lse;
    int hp;  // head pairs per KV group
};

// Shared memory map (bytes from the 1024-aligned base).
template <int D>
struct FwdSmem {
    static constexpr int DH = D / 64;                       // 64-column (128-byte) halves of d
    static constexpr uint32_t kQ = 0;                       // DH x [128 rows x 128 B]
    static constexpr uint32_t kQBytes = DH * 128 * 128;
    static constexpr uint32_t kKHalf = kBS * 128;           // one 64-column half of a K or V block
    static constexpr uint32_t kKV = kQ + kQBytes;           // stages x (K: DH halves, V: DH halves)
    static constexpr uint32_t kStageBytes = 2 * DH * kKHalf;
    static constexpr uint32_t kP = kKV + kStages * kStageBytes;   // 2 x [128 rows x 128 B]
    static constexpr uint32_t kPBytes = 128 * 128;
    static constexpr uint32_t kMask = kP + 2 * kPBytes;     // u64 [kMaxNB]
    static constexpr uint32_t kUnion = kMask + 8 * kMaxNB;  // u16 [kMaxNB + 1]
    static constexpr uint32_t kIdx = kUnion + 2 * (kMaxNB + 8);   // i16 [64][K<=64]
    static constexpr uint32_t kGl = kIdx + 2 * kTok * 64;   // f32 [64][K<=64]
    static constexpr uint32_t kNsel = kGl + 4 * kTok * 64;  // i32 [64]
    static constexpr uint32_t kBar = kNsel + 4 * kTok;      // mbarriers
    static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;  // tmem base, union count, abort flag
    static constexpr uint32_t kTotal = kMisc + 16;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, FwdTcArgs a) {
    using L = FwdSmem<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char* sQ = sm + L::kQ;
    unsigned char* sKV = sm + L::kKV;
    unsigned char* sP = sm + L::kP;
    unsigned long long* masks = reinterpret_cast<unsigned long long*>(sm + L::kMask);
    uint16_t* ulist = reinterpret_cast<uint16_t*>(sm + L::kUnion);
    int16_t* s_idx = reinterpret_cast<int16_t*>(sm + L::kIdx);
    float* s_gl = reinterpret_cast<float*>(sm + L::kGl);
    int* s_nsel = reinterpret_cast<int*>(sm + L::kNsel);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = bars + 1 + kStages;
    uint64_t* s_full = bars + 1 + 2 * kStages;
    uint64_t* p_full = s_full + 2;
    uint64_t* p_empty = p_full + 2;
    uint64_t* o_done = p_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
    int* n_union_slot = reinterpret_cast<int*>(sm + L::kMisc + 4);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 8);

    const Shape& sh = a.sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = sh.K, G = sh.G;
    // heaviest tiles (largest tau, longest union) first
    const int per_tau = sh.B * sh.Hkv * a.hp;
    const int tau = sh.nT - 1 - (int)(blockIdx.x / per_tau);
    const int rem = (int)(blockIdx.x % per_tau);
    const int hpi = rem % a.hp;
    const int bg = rem / a.hp;
    const int b = bg / sh.Hkv, g = bg % sh.Hkv;
    const int h0 = g * G + 2 * hpi;
    const bool h1_valid = 2 * hpi + 1 < G;
    const int h1 = h1_valid ? h0 + 1 : h0;
    const int64_t row0 = (int64_t)bg * sh.T + (int64_t)tau * kTok;   // first selection row of the tile

    if (tid == 0) {
        for (int i = 0; i < L::kNumBars; ++i) {
            uint64_t* bar = &bars[i];
            mbar_init(bar, (bar == &p_full[0] || bar == &p_full[1]) ? 4u : 1u);   // p_full: one arrive per softmax warp
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    // ---- the tile's selections: per-block token masks, per-token lists ----
    for (int j = tid; j < tau; j += kThreads) masks[j] = 0ull;
    if (tid < kTok) s_nsel[tid] = a.nsel[row0 + tid];
    __syncthreads();
    for (int e = tid; e < kTok * K; e += kThreads) {
        const int r = e / K, s = e - r * K;
        const int n = s_nsel[r];
        int j = -1;
        float lg = 0.f;
        if (s < n) {
            j = a.idx[(row0 + r) * K + s];
            lg = a.gl[(row0 + r) * K + s];
            if ((unsigned)j < (unsigned)tau) atomicOr(&masks[j], 1ull << r); else j = -1;
        }
        s_idx[r * K + s] = (int16_t)j;
        s_gl[r * K + s] = lg;
    }
    __syncthreads();
    if (warp == 0) {
        int cnt = 0;
        for (int base = 0; base < tau; base += 32) {
            const int j = base + lane;
            const bool nz = j < tau && masks[j] != 0ull;
            const uint32_t bal = __ballot_sync(0xffffffffu, nz);
            if (nz) ulist[cnt + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)j;
            cnt += __popc(bal);
        }
        if (lane == 0) {
            ulist[cnt] = (uint16_t)tau;
            *n_union_slot = cnt + 1;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int n = *n_union_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer ---
        if (lane == 0) {
            tc::prefetch_tmap(&tm_q);
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(q_full, L::kQBytes);
            const int qr0 = (int)(((int64_t)b * sh.Hq + h0) * sh.T + (int64_t)tau * kTok);
            const int qr1 = (int)(((int64_t)b * sh.Hq + h1) * sh.T + (int64_t)tau * kTok);
#pragma unroll
            for (int dh = 0; dh < L::DH; ++dh) {
                tc::tma_load_2d(sQ + dh * 128 * 128, &tm_q, dh * 64, qr0, q_full);
                tc::tma_load_2d(sQ + dh * 128 * 128 + 64 * 128, &tm_q, dh * 64, qr1, q_full);
            }
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int s = j % kStages;
                if (j >= kStages && !tc::wait_bar(&kv_empty[s], (uint32_t)((j / kStages - 1) & 1), abort)) break;
                const int blk = ulist[j];
                const int kr = (int)((int64_t)bg * sh.T + (int64_t)blk * kBS);
                unsigned char* st = sKV + s * L::kStageBytes;
                mbar_arrive_expect_tx(&kv_full[s], L::kStageBytes);
#pragma unroll
                for (int dh = 0; dh < L::DH; ++dh) {
                    tc::tma_load_2d(st + dh * L::kKHalf, &tm_k, dh * 64, kr, &kv_full[s]);
                    tc::tma_load_2d(st + (L::DH + dh) * L::kKHalf, &tm_v, dh * 64, kr, &kv_full[s]);
                }
                ++issued;
            }
            if (*abort) {
                // let the loads this thread started land before the CTA exits
                for (int j = issued - kStages; j < issued; ++j)
                    if (j >= 0) tc::drain_wait(&kv_full[j % kStages], (uint32_t)((j / kStages) & 1));
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kBS, false, false);
            constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, D, false, true);
            const uint32_t qa = smem_u32(sQ), kva = smem_u32(sKV), pa = smem_u32(sP);
            bool ok = tc::wait_bar(q_full, 0u, abort);
            tc::fence_after_sync();
            for (int j = 0; ok && j <= n; ++j) {
                if (j < n) {
                    const int s = j % kStages;
                    if (!tc::wait_bar(&kv_full[s], (uint32_t)((j / kStages) & 1), abort)) break;
                    tc::fence_after_sync();
                    const uint32_t kaddr = kva + s * L::kStageBytes;
                    const uint32_t d_s = tmem + (uint32_t)((j & 1) * kBS);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk & 3) * 32);     // 16 columns = 32 bytes
                        const uint64_t ad = tc::smem_desc_sw128(qa + (kk >> 2) * 128 * 128 + off, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(kaddr + (kk >> 2) * L::kKHalf + off, 16, 1024);
                        tc::mma_ss(d_s, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    tc::mma_commit(&s_full[j & 1]);
                }
                if (j >= 1) {
                    const int jp = j - 1;
                    if (!tc::wait_bar(&p_full[jp & 1], (uint32_t)((jp >> 1) & 1), abort)) break;
                    tc::fence_after_sync();
                    const int sp = jp % kStages;
                    const uint32_t vaddr = kva + sp * L::kStageBytes + L::DH * L::kKHalf;
                    const uint32_t paddr = pa + (jp & 1) * L::kPBytes;
#pragma unroll
                    for (int kk = 0; kk < kBS / 16; ++kk) {
                        const uint64_t ad = tc::smem_desc_sw128(paddr + kk * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(vaddr + kk * 16 * 128, L::kKHalf, 1024);
                        tc::mma_ss(tmem + 128, ad, bd, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&p_empty[jp & 1]);
                    tc::mma_commit(&kv_empty[sp]);
                    if (jp == n - 1) tc::mma_commit(o_done);
                }
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax + epilogue ---
        const int r = (warp - 4) * 32 + lane;      // tile row == TMEM lane
        const int tok = r & (kTok - 1);
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float qk = sh.scale * kLog2e;
        const int my_n = s_nsel[tok];
        const int16_t* my_idx = s_idx + tok * K;
        const float* my_gl = s_gl + tok * K;
        float m = -INFINITY, l = 0.f;
        int ptr = 0;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int blk = ulist[j];
            if (!tc::warp_wait_bar(&s_full[j & 1], (uint32_t)((j >> 1) & 1), abort)) { ok = false; break; }
            tc::fence_after_sync();
            uint32_t sr[kBS];
#pragma unroll
            for (int c = 0; c < kBS / 16; ++c) tc::tmem_ld16(lane_base + (uint32_t)((j & 1) * kBS + c * 16), sr + c * 16);
            tc::tmem_wait_ld();

            bool act;
            int kmax;
            float lg = 0.f;
            if (blk == tau) {
                act = true;
                kmax = tok;
            } else {
                act = ptr < my_n && my_idx[ptr] == blk;
                if (act) { lg = my_gl[ptr] * kLog2e; ++ptr; }
                kmax = kBS - 1;
            }
            float x[kBS];
            float mx = -INFINITY;
#pragma unroll
            for (int k = 0; k < kBS; ++k) {
                x[k] = (act && k <= kmax) ? fmaf(__uint_as_float(sr[k]), qk, lg) : -INFINITY;
                mx = fmaxf(mx, x[k]);
            }
            // lazy maximum: rescale O only when the new maximum exceeds the one in use by > 8
            float corr = 1.f;
            bool resc = false;
            if (mx > -INFINITY) {
                if (m == -INFINITY) {
                    m = mx;                      // O row is still exactly zero: nothing to rescale
                } else if (mx > m + 8.f) {
                    corr = exp2f(m - mx);
                    m = mx;
                    resc = true;
                }
            }
            if (__any_sync(0xffffffffu, resc)) {
                // the previous P V must be complete before O is rescaled in place
                if (!tc::warp_wait_bar(&p_empty[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t orr[16];
                    tc::tmem_ld16(lane_base + 128 + c * 16, orr);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                    tc::tmem_st16(lane_base + 128 + c * 16, orr);
                }
                tc::tmem_wait_st();
                l *= corr;
            }
            float psum = 0.f;
            uint32_t pk[kBS / 2];
#pragma unroll
            for (int k = 0; k < kBS; k += 2) {
                const float p0 = (x[k] == -INFINITY) ? 0.f : exp2f(x[k] - m);
                const float p1 = (x[k + 1] == -INFINITY) ? 0.f : exp2f(x[k + 1] - m);
                psum += p0 + p1;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                pk[k / 2] = *reinterpret_cast<uint32_t*>(&h2);
            }
            l += psum;
            // P buffer j&1 was last read by P V of block j-2
            if (j >= 2 && !tc::warp_wait_bar(&p_empty[j & 1], (uint32_t)(((j - 2) >> 1) & 1), abort)) { ok = false; break; }
            unsigned char* prow = sP + (j & 1) * L::kPBytes;
#pragma unroll
            for (int c = 0; c < kBS / 8; ++c) {
                const uint32_t off = tc::sw128_offset(r, c * 8);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(prow + off)),
                             "r"(pk[c * 4 + 0]), "r"(pk[c * 4 + 1]), "r"(pk[c * 4 + 2]), "r"(pk[c * 4 + 3])
                             : "memory");
            }
            tc::fence_async_shared();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&p_full[j & 1]);
        }
        if (ok && tc::warp_wait_bar(o_done, 0u, abort)) {
            tc::fence_after_sync();
            const int head = (r < kTok) ? h0 : h1;
            const bool write = r < kTok || h1_valid;
            const int64_t orow = ((int64_t)b * sh.Hq + head) * sh.T + (int64_t)tau * kTok + tok;
            const float inv = 1.f / l;
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
                uint32_t orr[16];
                tc::tmem_ld16(lane_base + 128 + c * 16, orr);
                tc::tmem_wait_ld();
                uint32_t packed[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(orr[2 * e]) * inv,
                                                              __uint_as_float(orr[2 * e + 1]) * inv);
                    packed[e] = *reinterpret_cast<uint32_t*>(&h2);
                }
                if (write) {
                    uint4* dst = reinterpret_cast<uint4*>(a.o + orow * D + c * 16);
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                }
            }
            if (write) a.lse[orow] = (m + log2f(l)) * kLn2;
        } else {
            // a wait gave up: leave a visibly invalid row instead of stale data
            const int head = (r < kTok) ? h0 : h1;
            if (r < kTok || h1_valid) {
                const int64_t orow = ((int64_t)b * sh.Hq + head) * sh.T + (int64_t)tau * kTok + tok;
                for (int c = 0; c < D; ++c) a.o[orow * D + c] = __float2bfloat16(__int_as_float(0x7fc00000));
                a.lse[orow] = __int_as_float(0x7fc00000);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t run_fwd_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                       const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!encode_bf16_2d(&mq, q, (uint64_t)s.B * s.Hq * s.T, D, 64) ||
        !encode_bf16_2d(&mk, k, (uint64_t)s.B * s.Hkv * s.T, D, kBS) ||
        !encode_bf16_2d(&mv, v, (uint64_t)s.B * s.Hkv * s.T, D, kBS))
        return cudaErrorInvalidValue;
    const size_t smem = FwdSmem<D>::kTotal + 1024;
    auto kern = fwd_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    FwdTcArgs a{s, idx, gl, nsel, static_cast<__nv_bfloat16*>(o), lse, (s.G + 1) / 2};
    const int64_t grid = (int64_t)s.B * s.Hkv * s.nT * a.hp;
    {
        KernelTimer kt("fwd_tc", st);
        kern<<<(unsigned)grid, kThreads, smem, st>>>(mq, mk, mv, a);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace

// cuTensorMapEncodeTiled is a driver entry point; it is looked up through the
// runtime so that the library does not link libcuda (and still loads, e.g. for
// argument checking, on machines without a driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    const EncodeTiledFn fn = encode_tiled_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool fwd_tc_supported(const Shape& s) {
    return s.dtype == SAS_DT_BF16 && s.D == 128 && s.bs == kBS && s.NB <= kMaxNB && s.K <= 64 && s.G <= 8 &&
           s.q_offset == 0 && s.T % kBS == 0 && (int64_t)s.B * s.Hq * s.T < ((int64_t)1 << 31);
}

cudaError_t launch_fwd_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                          const float* gl, const int32_t* nsel, void* o, float* lse, cudaStream_t st) {
    return run_fwd_tc<128>(s, q, k, v, idx, gl, nsel, o, lse, st);
}

cudaError_t read_fwd_tc_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

}  // namespace sas
