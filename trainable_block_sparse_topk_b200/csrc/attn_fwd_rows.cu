// attn_fwd_rows.cu -- gated block-sparse forward on the sm_100a tensor cores,
// key-block-centric over gathered rows.
//
// The forward (SAS study note 2-2 gated-attention eq.; arXiv text 4) is
//   o = softmax(a) V, a_j = scale q.k_j + log g_blk(j) on kept blocks, a_j =
//   scale q.k_j on the causal current block.
// Each token keeps its own K blocks, so a query tile shares few blocks; here
// every key block j instead gathers exactly the (token, head) rows that attend
// it (its own tile causally, and the later tokens whose selection kept j, from
// the column bitmap), in chunks of 128 rows, so every MMA row is a kept row.
// Two passes over the same row streams:
//   pass A (kOut = false): S = Q K_j^T, per row the maximum of a over the
//     block, combined across blocks with an atomic max on order-preserving
//     keys -> M (log2 units);
//   pass B (kOut = true):  S again, P = 2^(a log2 e - M) (<= 1), the row sums
//     l += sum P (fp32 atomics) and O += P V_j (M=128 rows, N=d, K=64 keys)
//     read back from TMEM, staged per row in shared memory and added into an
//     fp32 accumulator by bulk-copy reductions (whole lines at L2).
// A finalize kernel writes o = O / l and the row log-sum-exp M ln2 + ln l.
// Executed MMA work is 6 d FLOP per kept (query head, key) pair (the S
// product twice) with no masked rows, against 4 d in the definition.
//
// Roles (256 threads): warps 0 and 3 gather rows (even / odd chunks) with TMA
// tile::gather4 into two 128-byte-swizzled Q stages; warp 0 also loads K_j
// (and V_j) by TMA; warp 1 lane 0 issues the MMAs; warp 2 owns TMEM; warps 4-7
// compute (thread = row = TMEM lane). No TMA multicast is used.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sas {

namespace {

constexpr int kThreads = 256;
constexpr int kBS = 64;
constexpr int kRows = 128;
constexpr int kD = 128;

struct FwdRowsArgs {
    CUtensorMap tm_q;     // q [B*Hq*T, d], one-row boxes of 64 columns, 128-byte swizzle (gather4)
    Shape sh;
    const int32_t* idx;
    const float* gl;
    const int32_t* nsel;
    const uint64_t* maskT;
    uint32_t* rowmax;     // [B*Hq*T] order-preserving key of the row maximum of a (log2 units)
    float* l_acc;         // [B*Hq*T]
    float* o_acc;         // [B*Hq*T, d]
    int tpc;              // tokens per chunk = 128 / G
};

template <bool kOut>
struct RowsSmem {
    static constexpr uint32_t kK = 0;                              // K_j: 2 halves x [64 x 128 B]
    static constexpr uint32_t kV = 16384;                          // V_j (pass B)
    static constexpr uint32_t kStage = kOut ? 32768 : 16384;       // 2 x Q [2 x 128 x 128 B]
    static constexpr uint32_t kStageBytes = 32768;
    static constexpr uint32_t kP = kStage + 2 * kStageBytes;       // P [128 x 128 B] (pass B)
    static constexpr uint32_t kOst = kP + (kOut ? 16384 : 0);      // O rows, fp32, kOstRow apart (pass B)
    static constexpr uint32_t kOstRow = kD * 4 + 16;               // padded: conflict-free 16-byte stores
    static constexpr uint32_t kMeta = kOst + (kOut ? kRows * kOstRow : 0);  // 4 x per-chunk metadata
    static constexpr uint32_t kMetaBytes = 4 * 512 + 16;           // tok_t, tok_lg, row_m, qoff, ntok
    static constexpr uint32_t kBar = kMeta + 4 * kMetaBytes;
    static constexpr int kNumBars = 16;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;         // tmem base, token count, abort
    static constexpr uint32_t kColW = kMisc + 16;                  // u64 [nT] bitmap column, then i32 [nT] prefix
    static constexpr uint32_t kTmemCols = kOut ? 512 : 128;
    static uint32_t total(int nT) { return kColW + 12 * (uint32_t)nT + 16; }
};

struct RowMeta {
    int* tok_t;
    float* tok_lg;
    float* row_m;
    int* qoff;
    int* ntok;
    __device__ explicit RowMeta(unsigned char* p)
        : tok_t(reinterpret_cast<int*>(p)),
          tok_lg(reinterpret_cast<float*>(p + 512)),
          row_m(reinterpret_cast<float*>(p + 1024)),
          qoff(reinterpret_cast<int*>(p + 1536)),
          ntok(reinterpret_cast<int*>(p + 2048)) {}
};

__device__ __forceinline__ float key_to_float(uint32_t k) {
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

template <bool kOut>
__global__ void __launch_bounds__(kThreads, kOut ? 1 : 2)
fwd_rows_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ FwdRowsArgs a) {
    using L = RowsSmem<kOut>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* st_full = bars + 1;     // [2]: the loader's arrive + the gather bytes
    uint64_t* st_empty = bars + 3;    // [2] MMA commit + 4 compute-warp arrivals
    uint64_t* s_full = bars + 5;      // [2]
    uint64_t* s_empty = bars + 7;     // [2] pass A: 4 arrivals (compute warps)
    uint64_t* p_full = bars + 9;      // pass B: 4 arrivals
    uint64_t* p_empty = bars + 10;
    uint64_t* o_full = bars + 11;     // [2]
    uint64_t* o_empty = bars + 13;    // [2] 4 arrivals
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
    int* ntok_slot = reinterpret_cast<int*>(sm + L::kMisc + 4);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 8);

    const Shape& sh = a.sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = sh.G, K = sh.K, T = sh.T;
    const int ngroups = sh.B * sh.Hkv;
    const int j = (int)(blockIdx.x / ngroups);
    const int bg = (int)(blockIdx.x % ngroups);
    const int b = bg / sh.Hkv, g = bg % sh.Hkv;
    const int tpc = a.tpc;
    const uint64_t* col = a.maskT + ((int64_t)bg * sh.NB + j) * sh.nT;
    unsigned long long* colw = reinterpret_cast<unsigned long long*>(sm + L::kColW);
    int* pre = reinterpret_cast<int*>(sm + L::kColW + 8 * sh.nT);

    if (tid == 0) {
        for (int i = 0; i < L::kNumBars; ++i) {
            uint64_t* bar = &bars[i];
            uint32_t cnt = 1;
            if (bar == &s_empty[0] || bar == &s_empty[1] || bar == p_full || bar == &o_empty[0] || bar == &o_empty[1])
                cnt = 4;
            // a stage is refilled only after the MMA has read its rows and the
            // compute warps have waited for it: its phases then cannot run two
            // ahead of any waiter
            if (bar == &st_empty[0] || bar == &st_empty[1]) cnt = 5;
            mbar_init(bar, cnt);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(tmem_slot, L::kTmemCols);
        tc::tmem_relinquish();
    }
    // token stream of block j: its own 64 tokens, then later tokens that kept j
    for (int tau = tid; tau < sh.nT; tau += kThreads) colw[tau] = tau > j ? col[tau] : 0ull;
    __syncthreads();
    if (warp == 0) {
        const int per = (sh.nT + 31) / 32;
        const int t0 = lane * per, t1 = min(t0 + per, sh.nT);
        int sum = 0;
        for (int tau = t0; tau < t1; ++tau) sum += __popcll(colw[tau]);
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        int run = kBS + inc - sum;
        for (int tau = t0; tau < t1; ++tau) {
            pre[tau] = run;
            run += __popcll(colw[tau]);
        }
        if (lane == 31) *ntok_slot = kBS + inc;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ntok_total = *ntok_slot;
    const int nc = (ntok_total + tpc - 1) / tpc;
    const uint32_t sbase = smem_u32(sm);

    if (warp == 0 || warp == 3) {
        // ---------------------------------------------------------- loaders ---
        const int L0 = warp == 0 ? 0 : 1;
        unsigned char* stq = sm + L::kStage + L0 * L::kStageBytes;
        if (warp == 0 && lane == 0) {
            tc::prefetch_tmap(&tm_k);
            if (kOut) tc::prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(kv_full, kOut ? 32768u : 16384u);
            const int kr = (int)((int64_t)bg * T + (int64_t)j * kBS);
            for (int h = 0; h < 2; ++h) {
                tc::tma_load_2d(sm + L::kK + h * 8192, &tm_k, h * 64, kr, kv_full);
                if (kOut) tc::tma_load_2d(sm + L::kV + h * 8192, &tm_v, h * 64, kr, kv_full);
            }
        }
        auto token_at = [&](int s) -> int {
            if (s < kBS) return j * kBS + s;
            int lo = j + 1, hi = sh.nT - 1;      // last tile with pre[tile] <= s
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (pre[mid] <= s) lo = mid; else hi = mid - 1;
            }
            uint64_t w = colw[lo];
            for (int r = s - pre[lo]; r > 0; --r) w &= w - 1ull;
            return lo * kBS + __ffsll((long long)w) - 1;
        };
        auto prep = [&](int c) {
            RowMeta meta(sm + L::kMeta + (c & 3) * L::kMetaBytes);
            const int n = min(tpc, ntok_total - c * tpc);
            if (lane == 0) *meta.ntok = n;
            for (int i = lane; i < n; i += 32) {
                const int t = token_at(c * tpc + i);
                meta.tok_t[i] = t;
                float lg = 0.f;
                if ((t >> 6) != j) {
                    // log-gate of block j in the token's ascending kept list
                    const int64_t row = (int64_t)bg * T + t;
                    const int32_t* ir = a.idx + row * K;
                    const int ns = a.nsel[row];
                    int below = 0;
#pragma unroll 8
                    for (int s = 0; s < K; ++s) below += (s < ns && ir[s] < j) ? 1 : 0;
                    lg = a.gl[row * K + min(below, K - 1)];
                }
                meta.tok_lg[i] = lg;
            }
            __syncwarp();
            for (int i = lane; i < kRows; i += 32) {
                const int ti = i / G, h = i - ti * G;
                int qrow = -1;
                float m = 0.f;
                if (ti < n) {
                    qrow = (int)(((int64_t)b * sh.Hq + g * G + h) * T + meta.tok_t[ti]);
                    if (kOut) m = key_to_float(a.rowmax[qrow]);
                }
                meta.row_m[i] = m;
                meta.qoff[i] = qrow;
            }
            __syncwarp();
        };
        if (L0 < nc) prep(L0);
        for (int c = L0; c < nc; c += 2) {
            if (c >= 2 && !tc::warp_wait_bar(&st_empty[L0], (uint32_t)(((c >> 1) - 1) & 1), abort)) break;
            const int* qoff = RowMeta(sm + L::kMeta + (c & 3) * L::kMetaBytes).qoff;
            if (lane == 0) mbar_arrive_expect_tx(&st_full[L0], 32768u);
            __syncwarp();
            int rr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qrow = qoff[4 * lane + e];
                rr[e] = qrow >= 0 ? qrow : qoff[0];    // padding rows re-read a valid row; they are masked
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                tc::tma_gather4(stq + hh * 16384 + 4 * lane * 128, &a.tm_q, hh * 64, rr, &st_full[L0]);
            if (c + 2 < nc) prep(c + 2);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t id_s = tc::idesc_bf16_f32(128, kBS, false, false);
            constexpr uint32_t id_o = tc::idesc_bf16_f32(128, kD, false, true);
            const uint32_t ka = sbase + L::kK, va = sbase + L::kV, pa = sbase + L::kP;
            auto issue_s = [&](int c) {
                const uint32_t qa = sbase + L::kStage + (c & 1) * L::kStageBytes;
                const uint32_t ds = tmem + (uint32_t)((c & 1) * kBS);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t offk = (kk >> 2) * 8192 + (kk & 3) * 32;
                    tc::mma_ss(ds, tc::smem_desc_sw128(qa + off, 16, 1024), tc::smem_desc_sw128(ka + offk, 16, 1024),
                               id_s, kk > 0);
                }
                tc::mma_commit(&s_full[c & 1]);
                tc::mma_commit(&st_empty[c & 1]);     // Q of the stage is read only by S
            };
            bool ok = tc::wait_bar(kv_full, 0u, abort);
            if (!kOut) {
                for (int c = 0; ok && c < nc; ++c) {
                    if (!tc::wait_bar(&st_full[c & 1], (uint32_t)((c >> 1) & 1), abort)) break;
                    if (c >= 2 && !tc::wait_bar(&s_empty[c & 1], (uint32_t)(((c >> 1) - 1) & 1), abort)) break;
                    tc::fence_after_sync();
                    issue_s(c);
                }
            } else {
                // S of the next chunk (TMEM double buffer, at most one chunk ahead),
                // then O of the current chunk once P is in shared memory and its
                // O buffer has been read back.
                int s_next = 0, c = 0;
                uint64_t t0 = global_ns();
                while (ok && c < nc) {
                    bool progressed = false;
                    if (s_next < nc && s_next <= c + 1 &&
                        mbar_test_wait(&st_full[s_next & 1], (uint32_t)((s_next >> 1) & 1))) {
                        tc::fence_after_sync();
                        issue_s(s_next);
                        ++s_next;
                        progressed = true;
                    }
                    if (mbar_test_wait(p_full, (uint32_t)(c & 1)) &&
                        (c < 2 || mbar_test_wait(&o_empty[c & 1], (uint32_t)(((c >> 1) - 1) & 1)))) {
                        tc::fence_after_sync();
                        const uint32_t d_o = tmem + 128 + (uint32_t)((c & 1) * kD);
#pragma unroll
                        for (int kk = 0; kk < kBS / 16; ++kk)
                            tc::mma_ss(d_o, tc::smem_desc_sw128(pa + kk * 32, 16, 1024),
                                       tc::smem_desc_sw128(va + kk * 2048, 8192, 1024), id_o, kk > 0);
                        tc::mma_commit(&o_full[c & 1]);
                        tc::mma_commit(p_empty);
                        ++c;
                        progressed = true;
                    }
                    if (progressed) {
                        t0 = global_ns();
                    } else if (*abort) {
                        ok = false;
                    } else if (global_ns() - t0 > 1000000000ull) {
                        *abort = 1;
                        atomicAdd(&g_sas_wait_timeouts, 1u);
                        ok = false;
                    }
                }
            }
        }
    } else if (warp >= 4) {
        // ----------------------------------------------------- compute warps ---
        const int r = (warp - 4) * 32 + lane;      // chunk row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float qk = sh.scale * kLog2e;
        bool ok = true;
        int prev_row = -1;
        // O of chunk c: TMEM -> this thread's padded shared-memory row -> one
        // 512-byte bulk add into the fp32 accumulator row. The row is reused
        // only after the previous bulk add of this thread has read it.
        const uint32_t orow = sbase + L::kOst + (uint32_t)r * L::kOstRow;
        auto o_epilogue = [&](int c) -> bool {
            if (!tc::warp_wait_bar(&o_full[c & 1], (uint32_t)((c >> 1) & 1), abort)) return false;
            tc::fence_after_sync();
            const uint32_t col0 = 128 + (uint32_t)((c & 1) * kD);
            tc::bulk_wait_read0();
#pragma unroll 1
            for (int cb = 0; cb < kD / 16; ++cb) {
                uint32_t v[16];
                tc::tmem_ld16(lane_base + col0 + cb * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(orow + (cb * 16 + e) * 4),
                                 "r"(v[e]), "r"(v[e + 1]), "r"(v[e + 2]), "r"(v[e + 3]) : "memory");
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&o_empty[c & 1]);
            if (prev_row >= 0) {
                tc::fence_async_shared();
                tc::bulk_reduce_add_f32(a.o_acc + (int64_t)prev_row * kD, orow, kD * 4);
                tc::bulk_commit();
            }
            return true;
        };
        for (int c = 0; c < nc; ++c) {
            const int st = c & 1;
            if (!tc::warp_wait_bar(&st_full[st], (uint32_t)((c >> 1) & 1), abort)) { ok = false; break; }
            RowMeta meta(sm + L::kMeta + (c & 3) * L::kMetaBytes);
            const int n = *meta.ntok;
            const int ti = r / G;
            const bool valid = ti < n;
            int kmax = -1;
            float lg2 = 0.f, m = 0.f;
            int qrow = -1;
            if (valid) {
                const int t = meta.tok_t[ti];
                kmax = ((t >> 6) == j) ? (t & 63) : kBS - 1;
                lg2 = meta.tok_lg[ti] * kLog2e;
                m = meta.row_m[r];
                qrow = meta.qoff[r];
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&st_empty[st]);
            if (!tc::warp_wait_bar(&s_full[st], (uint32_t)((c >> 1) & 1), abort)) { ok = false; break; }
            tc::fence_after_sync();
            uint32_t sv[kBS];
#pragma unroll
            for (int cb = 0; cb < kBS / 16; ++cb) tc::tmem_ld16(lane_base + (uint32_t)(st * kBS + cb * 16), sv + cb * 16);
            tc::tmem_wait_ld();
            if (!kOut) {
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < kBS; ++k)
                    if (k <= kmax) mx = fmaxf(mx, fmaf(__uint_as_float(sv[k]), qk, lg2));
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&s_empty[st]);
                if (valid && mx > -INFINITY) atomicMax(a.rowmax + qrow, float_key(mx));
            } else {
                uint32_t pk[kBS / 2];
                float rs = 0.f;
                const float bias = lg2 - m;
#pragma unroll
                for (int k = 0; k < kBS; k += 2) {
                    const float p0 = (k <= kmax) ? exp2f(fmaf(__uint_as_float(sv[k]), qk, bias)) : 0.f;
                    const float p1 = (k + 1 <= kmax) ? exp2f(fmaf(__uint_as_float(sv[k + 1]), qk, bias)) : 0.f;
                    rs += p0 + p1;
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    pk[k / 2] = *reinterpret_cast<uint32_t*>(&hp);
                }
                if (valid) atomicAdd(a.l_acc + qrow, rs);
                if (c >= 1 && !tc::warp_wait_bar(p_empty, (uint32_t)((c - 1) & 1), abort)) { ok = false; break; }
#pragma unroll
                for (int cb = 0; cb < kBS / 8; ++cb) {
                    const uint32_t off = tc::sw128_offset(r, cb * 8);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + L::kP + off),
                                 "r"(pk[cb * 4]), "r"(pk[cb * 4 + 1]), "r"(pk[cb * 4 + 2]), "r"(pk[cb * 4 + 3])
                                 : "memory");
                }
                tc::fence_async_shared();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(p_full);
                if (c >= 1 && !o_epilogue(c - 1)) { ok = false; break; }
                prev_row = qrow;
            }
        }
        if (kOut && ok && nc > 0) o_epilogue(nc - 1);
        if (kOut) tc::bulk_wait0();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
}

// o = O / l (bf16) and attn_lse = M ln 2 + ln l, one warp per row.
__global__ void __launch_bounds__(256)
fwd_rows_finalize_kernel(int64_t rows, const uint32_t* __restrict__ rowmax, const float* __restrict__ l_acc,
                         const float* __restrict__ o_acc, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float l = l_acc[row];
    const float inv = 1.f / l;
    const float4 v = reinterpret_cast<const float4*>(o_acc + row * kD)[lane];
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * inv, v.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * inv, v.w * inv);
    uint2 packed = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    reinterpret_cast<uint2*>(o + row * kD)[lane] = packed;
    if (lane == 0) lse[row] = (key_to_float(rowmax[row]) + log2f(l)) * kLn2;
}

template <bool kOut>
cudaError_t launch_pass(const CUtensorMap& mk, const CUtensorMap& mv, const FwdRowsArgs& a, cudaStream_t st) {
    const size_t smem = RowsSmem<kOut>::total(a.sh.nT) + 1024;
    auto kern = fwd_rows_kernel<kOut>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)a.sh.B * a.sh.Hkv * a.sh.nT;
    kern<<<(unsigned)grid, kThreads, smem, st>>>(mk, mv, a);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

}  // namespace

bool fwd_rows_supported(const Shape& s) {
    return s.dtype == SAS_DT_BF16 && s.D == kD && s.bs == kBS && s.K <= 64 && s.G <= 8 && s.q_offset == 0 &&
           s.T % kBS == 0 && s.nT <= 1024 && (int64_t)s.B * s.Hq * s.T < ((int64_t)1 << 31);
}

size_t fwd_rows_ws_bytes(const Shape& s) {
    const size_t rows = (size_t)s.B * s.Hq * s.T;
    return 4 * rows + 4 * rows + 4 * rows * kD;
}

cudaError_t launch_fwd_rows(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                            const float* gl, const int32_t* nsel, const uint64_t* maskT, void* ws, void* o,
                            float* lse, cudaStream_t st) {
    const int64_t rows = (int64_t)s.B * s.Hq * s.T;
    uint32_t* rowmax = static_cast<uint32_t*>(ws);
    float* l_acc = reinterpret_cast<float*>(rowmax + rows);
    float* o_acc = l_acc + rows;
    CUtensorMap mk, mv;
    FwdRowsArgs a{};
    if (!encode_bf16_2d(&mk, k, (uint64_t)s.B * s.Hkv * s.T, kD, kBS) ||
        !encode_bf16_2d(&mv, v, (uint64_t)s.B * s.Hkv * s.T, kD, kBS) ||
        !encode_bf16_2d(&a.tm_q, q, (uint64_t)rows, kD, 1))
        return cudaErrorInvalidValue;
    a.sh = s;
    a.idx = idx;
    a.gl = gl;
    a.nsel = nsel;
    a.maskT = maskT;
    a.rowmax = rowmax;
    a.l_acc = l_acc;
    a.o_acc = o_acc;
    a.tpc = kRows / s.G;
    cudaError_t e = cudaMemsetAsync(ws, 0, fwd_rows_ws_bytes(s), st);
    if (e == cudaSuccess) e = launch_pass<false>(mk, mv, a, st);
    if (e == cudaSuccess) e = launch_pass<true>(mk, mv, a, st);
    if (e != cudaSuccess) return e;
    fwd_rows_finalize_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(rows, rowmax, l_acc, o_acc,
                                                                          static_cast<__nv_bfloat16*>(o), lse);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t read_fwd_rows_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

}  // namespace sas
