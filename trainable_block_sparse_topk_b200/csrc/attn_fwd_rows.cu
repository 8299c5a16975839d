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
//
// One pass: softmax is unchanged by any per-row shift M, so instead of the row
// maximum the shift is the row's own logit a_t = scale q_t.k_t (its key is
// always attended, with gate weight 1), computed by a small kernel first. Per
// chunk: S = Q K_j^T, P = 2^(a log2 e - M), the row sums l += sum P (fp32
// atomics) and O += P V_j (M=128 rows, N=d, K=64 keys), read back from TMEM,
// staged per row in shared memory and added into an fp32 accumulator by
// bulk-copy reductions (whole lines at L2). A finalize kernel writes o = O / l
// and the row log-sum-exp (M + log2 l) ln 2. Since P_t = 1, l >= 1: nothing
// underflows. A row whose largest logit exceeds a_t by more than ~80 (log2
// units) could overflow, so the finalize flags any row with l > 2^80 or a
// non-finite output and a CUDA-core kernel recomputes the flagged rows
// exactly (with the running maximum).
// Executed MMA work is the definition's 4 d FLOP per kept (query head, key)
// pair, with no masked rows.
//
// Roles (384 threads): warps 8, 11 and 10 gather rows (chunk c by loader
// c mod 3) with coalesced 16-byte cp.async copies into three 128-byte-swizzled
// Q stages (TMA tile::gather4 moves random rows at a fraction of that rate);
// with G = 1 the chunk metadata needs more shared memory and two stages (warps
// 8 and 11) are used. Warp 8 also loads K_j and V_j by TMA; warp 9 lane 0
// issues the MMAs; warp 10 owns TMEM; warps 4-7 form P (thread = row = TMEM
// lane) and warps 0-3 read O back and add it to the accumulator, so P of one
// chunk overlaps the output of the previous one. No TMA multicast is used.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sas {

namespace {

constexpr int kThreads = 384;   // epilogue 0-3, P 4-7, loaders 8 and 11, MMA 9, TMEM 10
constexpr int kBS = 64;
constexpr int kRows = 128;
constexpr int kD = 128;
constexpr size_t kMaxSmemPerBlock = 232448;   // 227 KB of opt-in dynamic shared memory per CTA

struct FwdRowsArgs {
    Shape sh;
    const __nv_bfloat16* q;   // [B*Hq*T, d]
    SelStream ss;         // per-block token streams: {t, log-gate}, the shift M of each head
    float* l_acc;         // [B*Hq*T]
    float* o_acc;         // [B*Hq*T, d]
    int tpc;              // tokens per chunk = 128 / G
    int meta_bytes;       // one metadata ring slot: tpc (16 + 4 rvs) bytes
    int* aborted;         // set when a CTA gave up on a wait (the finalize then writes NaN)
};

// kSt Q stages (3 when shared memory allows, else 2); the metadata ring has
// 2 kSt slots so each loader can request its next chunk's entries while it
// gathers the current one.
template <int kSt>
struct RowsSmem {
    static constexpr uint32_t kK = 0;                              // K_j: 2 halves x [64 x 128 B]
    static constexpr uint32_t kV = 16384;                          // V_j
    static constexpr uint32_t kStage = 32768;                      // kSt x Q [2 x 128 x 128 B]
    static constexpr uint32_t kStageBytes = 32768;
    static constexpr uint32_t kP = kStage + kSt * kStageBytes;     // P [128 x 128 B]
    static constexpr uint32_t kOst = kP + 16384;                   // O rows, fp32, kOstRow apart
    static constexpr uint32_t kOstRow = kD * 4 + 16;               // padded: conflict-free 16-byte stores
    static constexpr uint32_t kIds = kOst + kRows * kOstRow;       // i32 [4][128]: O accumulator row per chunk row
    static constexpr uint32_t kBar = kIds + 4 * kRows * 4;
    static constexpr int kMetaSlots = 2 * kSt;                     // chunk c -> slot c % kMetaSlots
    static constexpr int kNumBars = 14 + 4 * kSt;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;         // tmem base, stream length, first entry, abort
    static constexpr uint32_t kMeta = (kMisc + 16 + 15) & ~15u;    // metadata ring, meta_bytes per slot
    static constexpr uint32_t kTmemCols = 512;                     // S double [0,128), O double [128,384)
    static constexpr size_t total(int meta_bytes) { return kMeta + (size_t)kMetaSlots * meta_bytes; }
};

// One ring slot: the chunk's stream entries (token, log-gate) for tpc tokens,
// then each entry's per-head shift, copied in by the bulk-copy engine.
struct RowMeta {
    const int4* ent;
    const float* rv;
    __device__ RowMeta(const unsigned char* p, int tpc)
        : ent(reinterpret_cast<const int4*>(p)), rv(reinterpret_cast<const float*>(p + 16 * tpc)) {}
};

template <int kSt>
__global__ void __launch_bounds__(kThreads, 1)
fwd_rows_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ FwdRowsArgs a) {
    using L = RowsSmem<kSt>;
    constexpr int kMS = L::kMetaSlots;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* st_full = bars + 1;             // [kSt]: the loader's arrive once its copies have landed
    uint64_t* st_empty = st_full + kSt;       // [kSt] MMA commit + 4 compute-warp arrivals
    uint64_t* s_full = st_empty + kSt;        // [2]
    uint64_t* p_full = s_full + 2;            // 4 arrivals
    uint64_t* p_empty = p_full + 1;
    uint64_t* o_full = p_empty + 1;           // [2]
    uint64_t* o_empty = o_full + 2;           // [2] 4 arrivals
    uint64_t* meta_full = o_empty + 2;        // [kMS] ring slot c % kMS holds chunk c's stream entries (tx bytes)
    uint64_t* ids_full = meta_full + kMS;     // [4] 4 arrivals: chunk c's O rows are in ids[c & 3]
    uint64_t* mma_drain = ids_full + 4;       // every MMA of the CTA has completed
    int* ids = reinterpret_cast<int*>(sm + L::kIds);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
    int* ntok_slot = reinterpret_cast<int*>(sm + L::kMisc + 4);      // [2]: stream length, first entry
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 12);

    const Shape& sh = a.sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = sh.G, T = sh.T;
    // group-major CTA order: the CTAs running at once share one (b, kv head)
    // group, so its accumulator rows stay in L2 between their partial adds
    // (14B layer: 2-3% faster than key-block-major)
    const int j = (int)(blockIdx.x % sh.nT);
    const int bg = (int)(blockIdx.x / sh.nT);
    const int b = bg / sh.Hkv, g = bg % sh.Hkv;
    const int tpc = a.tpc;
    const int rvs = a.ss.rvs;

    if (tid == 0) {
        for (int i = 0; i < L::kNumBars; ++i) {
            uint64_t* bar = &bars[i];
            uint32_t cnt = 1;
            if (bar == p_full || bar == &o_empty[0] || bar == &o_empty[1]) cnt = 4;
            if (bar >= ids_full && bar < ids_full + 4) cnt = 4;
            // a stage is refilled only after the MMA has read its rows and the
            // compute warps have waited for it: its phases then cannot run two
            // ahead of any waiter
            if (bar >= st_empty && bar < st_empty + kSt) cnt = 5;
            if (bar >= st_full && bar < st_full + kSt) cnt = 33;   // 32 cp.async arrivals + the loader's
            mbar_init(bar, cnt);
        }
        ntok_slot[0] = a.ss.count[(int64_t)bg * sh.NB + j];   // tokens in block j's stream
        ntok_slot[1] = a.ss.base[(int64_t)bg * sh.NB + j];    // its first entry
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 10) {
        tc::tmem_alloc(tmem_slot, L::kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ntok_total = ntok_slot[0];
    const int64_t ebase = ntok_slot[1];
    const int nc = (ntok_total + tpc - 1) / tpc;
    const uint32_t sbase = smem_u32(sm);

    if (warp == 8 || warp == 11 || (kSt == 3 && warp == 10)) {
        // ---------------------------------------------------------- loaders ---
        // loader L0 fills stage L0 with chunks L0, L0 + kSt, ... (warp 10 joins
        // once it has allocated TMEM)
        const int L0 = warp == 8 ? 0 : warp == 11 ? 1 : 2;
        unsigned char* stq = sm + L::kStage + L0 * L::kStageBytes;
        if (warp == 8 && lane == 0) {
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(kv_full, 32768u);
            const int kr = (int)(sh.kv_index(bg) * T + (int64_t)j * kBS);
            for (int h = 0; h < 2; ++h) {
                tc::tma_load_2d(sm + L::kK + h * 8192, &tm_k, h * 64, kr, kv_full);
                tc::tma_load_2d(sm + L::kV + h * 8192, &tm_v, h * 64, kr, kv_full);
            }
        }
        // chunk c's stream entries -> ring slot c % kMS (bulk copies, completion on meta_full)
        int req_hi = -1, got_hi = -1;   // last chunk whose entries were requested / have landed
        auto request = [&](int c) {
            req_hi = c;
            if (lane == 0) {
                const int n = min(tpc, ntok_total - c * tpc);
                const int64_t e0 = ebase + (int64_t)c * tpc;
                const int s = c % kMS;
                unsigned char* slot = sm + L::kMeta + s * a.meta_bytes;
                const uint32_t be = 16u * (uint32_t)n, br = 4u * (uint32_t)(n * rvs);
                mbar_arrive_expect_tx(&meta_full[s], be + br);
                bulk_g2s(slot, a.ss.ent + e0, be, &meta_full[s]);
                bulk_g2s(slot + 16 * tpc, a.ss.rv + e0 * rvs, br, &meta_full[s]);
            }
        };
        if (L0 < nc) request(L0);
        for (int c = L0, k = 0; c < nc; c += kSt, ++k) {
            if (k >= 1 && !tc::warp_wait_bar(&st_empty[L0], (uint32_t)((k - 1) & 1), abort)) break;
            // slot (c + kSt) % kMS held chunk c - kSt, whose readers are done with it once its stage is released
            if (c + kSt < nc) request(c + kSt);
            if (!tc::warp_wait_bar(&meta_full[c % kMS], (uint32_t)((c / kMS) & 1), abort)) break;
            got_hi = c;
            const int4* ent = RowMeta(sm + L::kMeta + (c % kMS) * a.meta_bytes, tpc).ent;
            const int n = min(tpc, ntok_total - c * tpc);
            {
                // 16 lanes copy one 256-byte q row (16-byte pieces, coalesced), two
                // rows per instruction; piece p lands in d-half p / 8 at 16-byte
                // chunk p % 8 of the swizzled row. Padding rows re-read a valid row.
                const int p = lane & 15, hh = p >> 3, col = (p & 7) * 8;
#pragma unroll 4
                for (int i = 0; i < kRows / 2; ++i) {
                    const int row = 2 * i + (lane >> 4);
                    int ti = row / G, h = row - ti * G;
                    if (ti >= n) ti = 0, h = 0;
                    const int qrow = (int)(((int64_t)b * sh.Hq + g * G + h) * T + ent[ti].x);
                    tc::cp_async16(stq + hh * 16384 + tc::sw128_offset(row, col), a.q + (int64_t)qrow * kD + p * 8);
                }
            }
            // st_full completes once every lane's copies have landed (32 async
            // arrivals) and lane 0 has published the chunk's metadata; the MMA
            // thread fences the async proxy after its wait
            tc::cp_async_mbar_arrive_noinc(&st_full[L0]);
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&st_full[L0]);
        }
        tc::cp_async_wait_all();
        if (*abort && lane == 0) {
            // let the copies this warp started land before the CTA exits
            for (int c = got_hi < 0 ? L0 : got_hi + kSt; c <= req_hi; c += kSt)
                tc::drain_wait(&meta_full[c % kMS], (uint32_t)((c / kMS) & 1));
            if (warp == 8) tc::drain_wait(kv_full, 0u);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t id_s = tc::idesc_bf16_f32(128, kBS, false, false);
            constexpr uint32_t id_o = tc::idesc_bf16_f32(128, kD, false, true);
            const uint32_t ka = sbase + L::kK, va = sbase + L::kV, pa = sbase + L::kP;
            auto issue_s = [&](int c) {
                const uint32_t qa = sbase + L::kStage + (c % kSt) * L::kStageBytes;
                const uint32_t ds = tmem + (uint32_t)((c & 1) * kBS);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t offk = (kk >> 2) * 8192 + (kk & 3) * 32;
                    tc::mma_ss(ds, tc::smem_desc_sw128(qa + off, 16, 1024), tc::smem_desc_sw128(ka + offk, 16, 1024),
                               id_s, kk > 0);
                }
                tc::mma_commit(&s_full[c & 1]);
                tc::mma_commit(&st_empty[c % kSt]);   // Q of the stage is read only by S
            };
            bool ok = tc::wait_bar(kv_full, 0u, abort);
            {
                // S of the next chunk (TMEM double buffer, at most one chunk ahead),
                // then O of the current chunk once P is in shared memory and its
                // O buffer has been read back.
                int s_next = 0, c = 0;
                uint64_t t0 = global_ns();
                while (ok && c < nc) {
                    bool progressed = false;
                    if (s_next < nc && s_next <= c + 1 &&
                        mbar_test_wait(&st_full[s_next % kSt], (uint32_t)((s_next / kSt) & 1))) {
                        tc::fence_async_shared();
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
                    } else if (global_ns() - t0 > g_sas_wait_limit_ns) {
                        *abort = 1;
                        atomicAdd(&g_sas_wait_timeouts, 1u);
                        ok = false;
                    } else {
                        __nanosleep(40);   // back off: leave issue slots to the other warps of this SMSP
                    }
                }
            }
            tc::mma_commit(mma_drain);   // arrives once every MMA issued above has completed
        }
    } else if (warp >= 4 && warp < 8) {
        // --------------------------------------------------------- P warps ---
        const int r = (warp - 4) * 32 + lane;      // chunk row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float qk = sh.scale * kLog2e;
        for (int c = 0; c < nc; ++c) {
            const int stg = c % kSt, st = c & 1;    // Q stage, S buffer
            if (!tc::warp_wait_bar(&st_full[stg], (uint32_t)((c / kSt) & 1), abort)) break;
            const RowMeta meta(sm + L::kMeta + (c % kMS) * a.meta_bytes, tpc);
            const int n = min(tpc, ntok_total - c * tpc);
            const int ti = r / G, h = r - ti * G;
            const bool valid = ti < n;
            int kmax = -1;
            float lg2 = 0.f, m = 0.f;
            int qrow = -1;
            if (valid) {
                const int4 e = meta.ent[ti];
                const int t = e.x;
                kmax = ((t >> 6) == j) ? (t & 63) : kBS - 1;
                lg2 = __int_as_float(e.y) * kLog2e;
                m = meta.rv[ti * rvs + h];
                qrow = (int)(((int64_t)b * sh.Hq + g * G + h) * T + t);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&st_empty[stg]);
            if (!tc::warp_wait_bar(&s_full[st], (uint32_t)((c >> 1) & 1), abort)) break;
            tc::fence_after_sync();
            uint32_t sv[kBS];
#pragma unroll
            for (int cb = 0; cb < kBS / 16; ++cb) tc::tmem_ld16(lane_base + (uint32_t)(st * kBS + cb * 16), sv + cb * 16);
            tc::tmem_wait_ld();
            {
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
                // P of chunk c-1 has been consumed by its O product, which began only
                // after the epilogue warps were done with chunk c-3 -- and so with
                // the row ids of chunk c-4 that slot c & 3 held
                if (c >= 1 && !tc::warp_wait_bar(p_empty, (uint32_t)((c - 1) & 1), abort)) break;
                ids[(c & 3) * kRows + r] = qrow;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&ids_full[c & 3]);
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
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------ epilogue warps ---
        const int r = warp * 32 + lane;            // chunk row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        // O of chunk c: TMEM -> this thread's padded shared-memory row -> one
        // 512-byte bulk add into the fp32 accumulator row. The row is reused
        // only after the previous bulk add of this thread has read it.
        const uint32_t orow = sbase + L::kOst + (uint32_t)r * L::kOstRow;
        for (int c = 0; c < nc; ++c) {
            if (!tc::warp_wait_bar(&ids_full[c & 3], (uint32_t)((c >> 2) & 1), abort)) break;
            const int row_id = ids[(c & 3) * kRows + r];
            if (!tc::warp_wait_bar(&o_full[c & 1], (uint32_t)((c >> 1) & 1), abort)) break;
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
            if (row_id >= 0) {
                tc::fence_async_shared();
                tc::bulk_reduce_add_f32(a.o_acc + (int64_t)row_id * kD, orow, kD * 4);
                tc::bulk_commit();
            }
        }
        tc::bulk_wait0();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 10) {
        // TMEM is released only after the last MMA that writes it
        if (lane == 0) tc::drain_wait(mma_drain, 0u);
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
    if (tid == 0 && *abort) atomicExch(a.aborted, 1);
}

// M = scale log2e q_t.k_t for each of the G query heads of a (b, kv head, t)
// row, one warp per row: half a warp reads a 256-byte row (16 bytes a lane),
// both halves read k_t and heads 2u and 2u + 1 go to the two halves; the
// loads of all heads are issued before any sum. The warp also zeroes those
// rows' l and fp32 output accumulator rows, which the gathered-row kernel
// adds into.
__global__ void __launch_bounds__(256)
fwd_rows_shift_kernel(Shape sh, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      float* __restrict__ shift, float* __restrict__ l_acc, float* __restrict__ o_acc) {
    const int row = (int)(blockIdx.x * 8 + (threadIdx.x >> 5));   // (b * Hkv + g) * T + t
    const int lane = threadIdx.x & 31, sub = lane >> 4, li = lane & 15;
    if (row >= sh.rows()) return;
    const int bg = row / sh.T;
    const int t = row - bg * sh.T;
    const int b = bg / sh.Hkv, g = bg - b * sh.Hkv;
    const uint4 kv = *reinterpret_cast<const uint4*>(k + (sh.kv_index(bg) * sh.T + t) * kD + li * 8);
    uint4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {                      // G <= 8
        const int h = 2 * u + sub;
        x[u] = make_uint4(0u, 0u, 0u, 0u);
        if (h < sh.G)
            x[u] = *reinterpret_cast<const uint4*>(q + (((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + t) * kD + li * 8);
    }
    float c[8];
    load_vec<__nv_bfloat16, 8>(reinterpret_cast<const __nv_bfloat16*>(&kv), c);
    const float qk = sh.scale * kLog2e;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (2 * u >= sh.G) break;                      // warp-uniform
        float a[8];
        load_vec<__nv_bfloat16, 8>(reinterpret_cast<const __nv_bfloat16*>(&x[u]), a);
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = fmaf(a[e], c[e], d);
#pragma unroll
        for (int m = 8; m > 0; m >>= 1) d += __shfl_xor_sync(0xffffffffu, d, m);
        const int h = 2 * u + sub;
        if (li == 0 && h < sh.G) shift[((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + t] = d * qk;
    }
    for (int h = 0; h < sh.G; ++h) {
        const int64_t qrow = ((int64_t)b * sh.Hq + g * sh.G + h) * sh.T + t;
        reinterpret_cast<float4*>(o_acc + qrow * kD)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0) l_acc[qrow] = 0.f;
    }
}

// o = O / l (bf16) and attn_lse = (M + log2 l) ln 2, one warp per query-head
// row; each warp takes kRowsU rows per pass and issues all their loads before
// using any. Rows whose sum or output left the safe range are listed (as their
// (b, kv head, t) row) for the exact recompute instead.
constexpr int kRowsU = 4;

__global__ void __launch_bounds__(256)
fwd_rows_finalize_kernel(Shape sh, const float* __restrict__ shift, const float* __restrict__ l_acc,
                         const float* __restrict__ o_acc, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                         int32_t* __restrict__ list, int32_t* __restrict__ list_n, const int* __restrict__ aborted) {
    const int64_t rows = (int64_t)sh.B * sh.Hq * sh.T;
    if (*aborted) {
        // a CTA of the gathered-row kernel gave up on a wait: the accumulators
        // are incomplete, so every output row is marked invalid
        const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
        const __nv_bfloat16 nan = __float2bfloat16(__int_as_float(0x7fc00000));
        for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * kD; e += nthr) o[e] = nan;
        for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows; e += nthr)
            lse[e] = __int_as_float(0x7fc00000);
        return;
    }
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r0 = warp * kRowsU; r0 < rows; r0 += nwarps * kRowsU) {
        float4 v[kRowsU];
        float l[kRowsU];
#pragma unroll
        for (int u = 0; u < kRowsU; ++u) {
            const int64_t row = r0 + u;
            if (row >= rows) continue;
            v[u] = reinterpret_cast<const float4*>(o_acc + row * kD)[lane];
            l[u] = l_acc[row];
        }
#pragma unroll
        for (int u = 0; u < kRowsU; ++u) {
            const int64_t row = r0 + u;
            if (row >= rows) continue;                    // warp-uniform
            const bool fin = isfinite(v[u].x) && isfinite(v[u].y) && isfinite(v[u].z) && isfinite(v[u].w);
            const bool bad = __any_sync(0xffffffffu, !fin) || !(l[u] >= 0.5f && l[u] <= 0x1p80f);
            if (bad) {
                if (lane == 0) {
                    const int64_t bh = row / sh.T;
                    const int t = (int)(row % sh.T);
                    const int b = (int)(bh / sh.Hq), h = (int)(bh % sh.Hq);
                    list[atomicAdd(list_n, 1)] = (int32_t)(((int64_t)b * sh.Hkv + h / sh.G) * sh.T + t);
                }
                continue;
            }
            const float inv = 1.f / l[u];
            __nv_bfloat162 lo = __floats2bfloat162_rn(v[u].x * inv, v[u].y * inv);
            __nv_bfloat162 hi = __floats2bfloat162_rn(v[u].z * inv, v[u].w * inv);
            uint2 packed = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
            reinterpret_cast<uint2*>(o + row * kD)[lane] = packed;
            if (lane == 0) lse[row] = (shift[row] + log2f(l[u])) * kLn2;
        }
    }
}

// Workspace: shift [rows] f32 | list [rows] i32 | l [rows] f32 | O [rows, d] f32 | list count |
// abort flag | (256-aligned) the token streams
struct RowsWs {
    float* shift;
    int32_t* list;
    float* l_acc;
    float* o_acc;
    int32_t* list_n;
    RowsWs(void* ws, int64_t rows)
        : shift(static_cast<float*>(ws)),
          list(reinterpret_cast<int32_t*>(shift + rows)),
          l_acc(reinterpret_cast<float*>(list + rows)),
          o_acc(l_acc + rows),
          list_n(reinterpret_cast<int32_t*>(o_acc + rows * kD)) {}
    static size_t head_bytes(int64_t rows) { return (12 * (size_t)rows + 4 * (size_t)rows * kD + 16 + 255) & ~(size_t)255; }
};

}  // namespace

bool fwd_rows_supported(const Shape& s) {
    return s.dtype == SAS_DT_BF16 && s.D == kD && s.bs == kBS && s.K <= 64 && s.G <= 8 && s.q_offset == 0 &&
           s.T % kBS == 0 && s.nT <= 1024 && (int64_t)s.B * s.Hq * s.T < ((int64_t)1 << 31);
}

size_t fwd_rows_ws_bytes(const Shape& s) {
    return RowsWs::head_bytes((int64_t)s.B * s.Hq * s.T) + sel_stream_bytes(s, 1);
}

cudaError_t launch_fwd_rows(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                            const float* gl, const int32_t* nsel, const uint64_t* maskT, void* ws, void* o,
                            float* lse, cudaStream_t st) {
    const int64_t rows = (int64_t)s.B * s.Hq * s.T;
    const RowsWs w(ws, rows);
    CUtensorMap mk, mv;
    FwdRowsArgs a{};
    if (!encode_bf16_2d(&mk, k, (uint64_t)s.B * s.Hkvp * s.T, kD, kBS) ||
        !encode_bf16_2d(&mv, v, (uint64_t)s.B * s.Hkvp * s.T, kD, kBS))
        return cudaErrorInvalidValue;
    a.sh = s;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.ss = sel_stream_at(static_cast<unsigned char*>(ws) + RowsWs::head_bytes(rows), s, 1);
    a.l_acc = w.l_acc;
    a.o_acc = w.o_acc;
    a.tpc = kRows / s.G;
    a.aborted = w.list_n + 1;
    cudaError_t e = cudaMemsetAsync(w.list_n, 0, 2 * sizeof(int32_t), st);   // list count, abort flag
    if (e != cudaSuccess) return e;
    {
        KernelTimer kt("fwd_rows_shift", st);
        fwd_rows_shift_kernel<<<(unsigned)((s.rows() + 7) / 8), 256, 0, st>>>(s, a.q, static_cast<const __nv_bfloat16*>(k),
                                                                               w.shift, w.l_acc, w.o_acc);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    e = launch_sel_stream(s, maskT, idx, gl, nsel, w.shift, nullptr, 1, a.ss, st);
    if (e != cudaSuccess) return e;
    a.meta_bytes = a.tpc * (16 + 4 * a.ss.rvs);
    // three Q stages when they fit in shared memory (G >= 2), else two
    const size_t smem3 = RowsSmem<3>::total(a.meta_bytes) + 1024;
    const bool three = smem3 <= kMaxSmemPerBlock;
    const size_t smem = three ? smem3 : RowsSmem<2>::total(a.meta_bytes) + 1024;
    auto kern = three ? fwd_rows_kernel<3> : fwd_rows_kernel<2>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    {
        KernelTimer kt("fwd_rows", st);
        kern<<<(unsigned)((int64_t)s.B * s.Hkv * s.nT), kThreads, smem, st>>>(mk, mv, a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    {
        KernelTimer kt("fwd_rows_finalize", st);
        fwd_rows_finalize_kernel<<<(unsigned)std::min<int64_t>((rows + 8 * kRowsU - 1) / (8 * kRowsU), 148 * 16), 256, 0,
                                   st>>>(s, w.shift, w.l_acc, w.o_acc, static_cast<__nv_bfloat16*>(o), lse, w.list,
                                         w.list_n, a.aborted);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launches(1);
    return launch_fwd_simt_rows(s, q, k, v, idx, gl, nsel, w.list, w.list_n, o, lse, st);
}

cudaError_t set_fwd_rows_wait_limit(unsigned long long ns) {
    return cudaMemcpyToSymbol(g_sas_wait_limit_ns, &ns, sizeof(ns));
}

cudaError_t read_fwd_rows_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

}  // namespace sas
