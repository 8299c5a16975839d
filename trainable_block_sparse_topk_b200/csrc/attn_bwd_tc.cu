// attn_bwd_tc.cu -- gated block-sparse backward on the sm_100a tensor cores.
//
// Gradients of o = softmax(a) V with a_j = scale q.k_j + log g_blk(j) (SAS
// study note 2-2, 3-6 "keeps the selector gradient"; arXiv text 4):
//   P = exp(a - lse), dP = dO V^T, dS = P (dP - D) with D = rowsum(dO o),
//   dV += P^T dO, dK += scale dS^T q, dQ = scale dS K,
//   Gsum[row, slot] = sum of dS over the block's tokens and the group's heads
// (the gradient of the row's log-gate of that block; the score gradient is
// formed from it by the epilogue kernel).
//
// Tiling: key-block-centric. One CTA owns key block j of one (batch, KV
// group). It streams the (token, head) rows whose attention includes j -- the
// block's own 64 tokens (causally) and every later token whose selection kept
// j -- in chunks of 128 gathered rows (128/G tokens x G heads), so every MMA
// row is a kept row. The walk is laid out beforehand as a per-block token
// stream (stream.cu) whose entries carry each token's log-gate and kept-list
// slot and each row's lse and D; the CTA bulk-copies a chunk's entries into
// a ring two chunks ahead. Per chunk:
//   S = Q K_j^T and dP = dO V_j^T  (M=128 rows, N=64 keys, K=d)   -> TMEM
//   P, dS in the compute warps (thread = row = TMEM lane), Gsum per token
//   dV^T += dO^T P, dK^T += Q^T dS (M=d, N=64, K=128 rows)        -> TMEM
//   dQ = dS K_j (M=128 rows, N=d, K=64)                            -> TMEM
//   dQ rows are added into the fp32 accumulator with vector atomics, lanes
//   regrouped so that each warp-wide reduction covers whole L2 sectors.
// TMEM: S|dP double buffer [0,256), dQ [256,384), dV^T [384,448),
// dK^T [448,512). S/dP of chunk c+1 are computed while warps 4-7 build P/dS
// of chunk c and warps 0-3 read back and add dQ of chunk c-1.
//
// Roles (512 threads): warps 0-3 epilogue (dQ reductions, final dK/dV),
// warps 4-7 and 12-15 P/dS and Gsum for keys 0-31 and 32-63 of the block
// (thread = row = TMEM lane in every group), warps 8 and 11 gather each
// chunk's rows (rows 0-63 / 64-127) with coalesced 16-byte cp.async copies
// into the two 128-byte-swizzled Q/dO stages (TMA tile::gather4 moves random
// rows at a fraction of that rate; warp 8 also loads K_j, V_j by TMA), warp 9
// lane 0 issues the MMAs, warp 10 owns the TMEM allocation. No TMA multicast
// is used.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace sas {

namespace {

constexpr int kThreads = 512;   // epilogue warps 0-3, P/dS warps 4-7 and 12-15, loaders 8 and 11, MMA 9, TMEM 10
constexpr int kBS = 64;
constexpr int kRows = 128;
constexpr int kD = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDQ = 256, kColDV = 384, kColDK = 448;

struct BwdTcArgs {
    Shape sh;
    const __nv_bfloat16* q;
    const __nv_bfloat16* dO;
    SelStream ss;        // per-block token streams: {t, log-gate, slot}, then lse and D of each head
    float* dq_acc;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* gsum;
    float* dk32;         // per-query-head selection: fp32 dK, dV of each selection group
    float* dv32;         // ([B * Hkv, T, d], summed over the heads of a KV head later); else NULL
    int tpc;             // tokens per chunk = 128 / G
    int meta_bytes;      // one metadata ring slot: tpc (16 + 4 rvs) bytes
    int* aborted;        // set when a CTA gave up on a wait (the later kernels then write NaN)
};

struct BwdSmem {
    static constexpr uint32_t kK = 0;                          // K_j: 2 halves x [64 x 128 B]
    static constexpr uint32_t kV = 16384;                      // V_j
    static constexpr uint32_t kStage = 32768;                  // 2 x (Q [2 x 128 x 128 B] | dO [same])
    static constexpr uint32_t kStageBytes = 65536;
    static constexpr uint32_t kP = kStage + 2 * kStageBytes;   // P  [128 x 128 B]
    static constexpr uint32_t kDS = kP + 16384;                // dS [128 x 128 B]
    static constexpr uint32_t kGs = kDS + 16384;               // per-token Gsum [2][128] f32
    static constexpr uint32_t kIds = kGs + 1024;               // i32 [2][128]: dQ accumulator row per chunk row
    static constexpr uint32_t kBar = kIds + 1024;
    static constexpr int kNumBars = 18;
    static constexpr uint32_t kMisc = kBar + 8 * kNumBars;     // tmem base, stream length, first entry, abort
    static constexpr uint32_t kMeta = (kMisc + 16 + 15) & ~15u;   // 4 x chunk stream entries (chunk c -> slot c & 3)
    static constexpr size_t total(int meta_bytes) { return kMeta + 4 * (size_t)meta_bytes; }
};

// One metadata ring slot: the chunk's stream entries (token, log-gate, slot of
// block j in the token's kept list) for tpc tokens, then per entry the lse and
// D of each of its G query heads; copied in by the bulk-copy engine.
struct ChunkMeta {
    const int4* ent;
    const float* rv;
    __device__ ChunkMeta(const unsigned char* p, int tpc)
        : ent(reinterpret_cast<const int4*>(p)), rv(reinterpret_cast<const float*>(p + 16 * tpc)) {}
};

__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ BwdTcArgs a) {
    using L = BwdSmem;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* kv_full = bars + 0;
    uint64_t* st_full = bars + 1;     // [2], the loader's arrive once its copies have landed
    uint64_t* st_empty = bars + 3;    // [2]
    uint64_t* s_full = bars + 5;      // [2]
    uint64_t* p_full = bars + 7;      // 8 arrivals (P/dS warps)
    uint64_t* p_empty = bars + 8;
    uint64_t* dq_full = bars + 9;
    uint64_t* dq_empty = bars + 10;   // 4 arrivals
    uint64_t* done = bars + 11;
    uint64_t* ids_full = bars + 12;   // [2] 4 arrivals: the chunk's dQ row ids are in ids[]
    uint64_t* meta_full = bars + 14;  // [4] ring slot c & 3 holds chunk c's stream entries (tx bytes)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc);
    int* ntok_slot = reinterpret_cast<int*>(sm + L::kMisc + 4);      // [2]: stream length, first entry
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 12);
    float* tok_gs = reinterpret_cast<float*>(sm + L::kGs);
    int* ids = reinterpret_cast<int*>(sm + L::kIds);

    const Shape& sh = a.sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = sh.G, K = sh.K, T = sh.T;
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
            if (bar == dq_empty || bar == &ids_full[0] || bar == &ids_full[1]) cnt = 4;
            if (bar == p_full) cnt = 8;
            // both loaders fill every stage: 32 cp.async arrivals + one arrive each
            if (bar == &st_full[0] || bar == &st_full[1]) cnt = 66;
            mbar_init(bar, cnt);
        }
        ntok_slot[0] = a.ss.count[(int64_t)bg * sh.NB + j];   // tokens in block j's stream
        ntok_slot[1] = a.ss.base[(int64_t)bg * sh.NB + j];    // its first entry
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 10) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int i = tid; i < 2 * kRows; i += kThreads) tok_gs[i] = 0.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ntok_total = ntok_slot[0];
    const int64_t ebase = ntok_slot[1];
    const int nc = (ntok_total + tpc - 1) / tpc;
    const uint32_t sbase = smem_u32(sm);

    if (warp == 8 || warp == 11) {
        // ---------------------------------------------------------- loaders ---
        // Both loaders gather every chunk (warp 8 rows 0-63, warp 11 rows
        // 64-127); loader w requests the stream entries of chunks c = w mod 2.
        const int w = warp == 8 ? 0 : 1;
        if (warp == 8 && lane == 0) {
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(kv_full, 32768);
            const int kr = (int)(sh.kv_index(bg) * T + (int64_t)j * kBS);
            for (int h = 0; h < 2; ++h) {
                tc::tma_load_2d(sm + L::kK + h * 8192, &tm_k, h * 64, kr, kv_full);
                tc::tma_load_2d(sm + L::kV + h * 8192, &tm_v, h * 64, kr, kv_full);
            }
        }
        // chunk c's stream entries -> ring slot c & 3 (bulk copies, completion on meta_full)
        int req_hi = -1, got_hi = -1;   // last chunk requested by this loader / whose entries have landed
        auto request = [&](int c) {
            req_hi = c;
            if (lane == 0) {
                const int n = min(tpc, ntok_total - c * tpc);
                const int64_t e0 = ebase + (int64_t)c * tpc;
                unsigned char* slot = sm + L::kMeta + (c & 3) * a.meta_bytes;
                const uint32_t be = 16u * (uint32_t)n, br = 4u * (uint32_t)(n * rvs);
                mbar_arrive_expect_tx(&meta_full[c & 3], be + br);
                bulk_g2s(slot, a.ss.ent + e0, be, &meta_full[c & 3]);
                bulk_g2s(slot + 16 * tpc, a.ss.rv + e0 * rvs, br, &meta_full[c & 3]);
            }
        };
        if (w < nc) request(w);
        for (int c = 0; c < nc; ++c) {
            if (c >= 2 && !tc::warp_wait_bar(&st_empty[c & 1], (uint32_t)(((c >> 1) - 1) & 1), abort)) break;
            // slot (c + 2) & 3 held chunk c - 2, whose readers are done with it once its stage is released
            if ((c & 1) == w && c + 2 < nc) request(c + 2);
            if (!tc::warp_wait_bar(&meta_full[c & 3], (uint32_t)((c >> 2) & 1), abort)) break;
            got_hi = c;
            const int4* ent = ChunkMeta(sm + L::kMeta + (c & 3) * a.meta_bytes, tpc).ent;
            const int n = min(tpc, ntok_total - c * tpc);
            unsigned char* stq = sm + L::kStage + (c & 1) * L::kStageBytes;
            unsigned char* stdo = stq + 32768;
            {
                // 16 lanes copy one 256-byte row (16-byte pieces, coalesced), two
                // rows per instruction, into the swizzled tile; row i's piece p
                // lands in d-half p / 8 at 16-byte chunk p % 8. Padding rows
                // re-read the chunk's first row (their P and dS are zero).
                const int p = lane & 15, hh = p >> 3, col = (p & 7) * 8;
#pragma unroll 4
                for (int i = 0; i < kRows / 4; ++i) {
                    const int row = w * (kRows / 2) + 2 * i + (lane >> 4);
                    int ti = row / G, h = row - ti * G;
                    if (ti >= n) ti = 0, h = 0;
                    const int64_t qrow = ((int64_t)b * sh.Hq + g * G + h) * T + ent[ti].x;
                    const uint32_t off = hh * 16384 + tc::sw128_offset(row, col);
                    tc::cp_async16(stq + off, a.q + qrow * kD + p * 8);
                    tc::cp_async16(stdo + off, a.dO + qrow * kD + p * 8);
                }
            }
            // st_full completes once both loaders' copies have landed (32 async
            // arrivals each) and each has arrived once; the MMA thread fences
            // the async proxy after its wait
            tc::cp_async_mbar_arrive_noinc(&st_full[c & 1]);
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&st_full[c & 1]);
        }
        tc::cp_async_wait_all();
        if (*abort && lane == 0) {
            // let the copies this warp started land before the CTA exits
            int c0 = got_hi + 1;
            if ((c0 & 1) != w) ++c0;
            for (int c = c0; c <= req_hi; c += 2) tc::drain_wait(&meta_full[c & 3], (uint32_t)((c >> 2) & 1));
            if (warp == 8) tc::drain_wait(kv_full, 0u);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t id_sp = tc::idesc_bf16_f32(128, kBS, false, false);   // S, dP
            constexpr uint32_t id_kv = tc::idesc_bf16_f32(128, kBS, true, true);     // dV^T, dK^T
            constexpr uint32_t id_dq = tc::idesc_bf16_f32(128, kD, false, true);     // dQ
            const uint32_t ka = sbase + L::kK, va = sbase + L::kV;
            const uint32_t pa = sbase + L::kP, dsa = sbase + L::kDS;
            auto issue_sdp = [&](int c) {
                const uint32_t qa = sbase + L::kStage + (c & 1) * L::kStageBytes, doa = qa + 32768;
                const uint32_t dsp = tmem + (uint32_t)((c & 1) * 128);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t offk = (kk >> 2) * 8192 + (kk & 3) * 32;
                    tc::mma_ss(dsp, tc::smem_desc_sw128(qa + off, 16, 1024), tc::smem_desc_sw128(ka + offk, 16, 1024),
                               id_sp, kk > 0);
                    tc::mma_ss(dsp + 64, tc::smem_desc_sw128(doa + off, 16, 1024),
                               tc::smem_desc_sw128(va + offk, 16, 1024), id_sp, kk > 0);
                }
                tc::mma_commit(&s_full[c & 1]);
            };
            bool ok = tc::wait_bar(kv_full, 0u, abort) && tc::wait_bar(&st_full[0], 0u, abort);
            tc::fence_async_shared();   // the stage was written by cp.async (generic proxy)
            tc::fence_after_sync();
            if (ok) issue_sdp(0);
            // Issue whichever step is ready: S/dP of the next chunk (TMEM double
            // buffer: at most one chunk ahead), dV/dK of the current chunk once
            // its P/dS are in shared memory, then its dQ once the previous dQ
            // has been read back.
            int sdp_next = 1, c = 0;
            bool kv_issued = false;
            uint64_t t0 = global_ns();
            while (ok && c < nc) {
                bool progressed = false;
                if (sdp_next < nc && sdp_next <= c + 1 &&
                    mbar_test_wait(&st_full[sdp_next & 1], (uint32_t)((sdp_next >> 1) & 1))) {
                    tc::fence_async_shared();
                    tc::fence_after_sync();
                    issue_sdp(sdp_next);
                    ++sdp_next;
                    progressed = true;
                }
                if (!kv_issued && mbar_test_wait(p_full, (uint32_t)(c & 1))) {
                    tc::fence_after_sync();
                    const uint32_t qa = sbase + L::kStage + (c & 1) * L::kStageBytes, doa = qa + 32768;
#pragma unroll
                    for (int kk = 0; kk < kRows / 16; ++kk) {
                        const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
                        tc::mma_ss(tmem + kColDV, tc::smem_desc_sw128(doa + kk * 2048, 16384, 1024),
                                   tc::smem_desc_sw128(pa + kk * 2048, 16384, 1024), id_kv, acc);
                        tc::mma_ss(tmem + kColDK, tc::smem_desc_sw128(qa + kk * 2048, 16384, 1024),
                                   tc::smem_desc_sw128(dsa + kk * 2048, 16384, 1024), id_kv, acc);
                    }
                    tc::mma_commit(&st_empty[c & 1]);   // the stage's Q and dO are no longer needed
                    kv_issued = true;
                    progressed = true;
                }
                if (kv_issued && (c == 0 || mbar_test_wait(dq_empty, (uint32_t)((c - 1) & 1)))) {
                    tc::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < kBS / 16; ++kk)
                        tc::mma_ss(tmem + kColDQ, tc::smem_desc_sw128(dsa + kk * 32, 16, 1024),
                                   tc::smem_desc_sw128(ka + kk * 2048, 8192, 1024), id_dq, kk > 0);
                    tc::mma_commit(dq_full);
                    tc::mma_commit(p_empty);
                    ++c;
                    kv_issued = false;
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
            tc::mma_commit(done);
        }
    } else if ((warp >= 4 && warp < 8) || warp >= 12) {
        // ------------------------------ P / dS warps (4 - 7: keys 0-31, 12 - 15: keys 32-63) ---
        const int r = (warp & 3) * 32 + lane;      // chunk row == TMEM lane
        const int hf = warp >= 12 ? 1 : 0;         // which 32 keys of the block
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float qk = sh.scale * kLog2e;
        for (int c = 0; c < nc; ++c) {
            const int st = c & 1;
            float* gs = tok_gs + st * kRows;
            int n = 0, gs_slot = -1, gs_tok = 0;
            bool fail = false;
            do {   // a wait that gives up leaves this block, not the chunk loop
                if (!tc::warp_wait_bar(&st_full[st], (uint32_t)((c >> 1) & 1), abort)) { fail = true; break; }
                const ChunkMeta meta(sm + L::kMeta + (c & 3) * a.meta_bytes, tpc);
                n = min(tpc, ntok_total - c * tpc);
                const int ti = r / G, h = r - ti * G;
                const bool valid = ti < n;
                int t = 0, kmax = -1;
                float lgl = 0.f, lse2 = 0.f, Dv = 0.f;
                bool diag = false;
                if (valid) {
                    const int4 e = meta.ent[ti];
                    t = e.x;
                    diag = (t >> 6) == j;
                    kmax = diag ? (t & 63) : kBS - 1;
                    lgl = __int_as_float(e.y);
                    lse2 = meta.rv[ti * rvs + 2 * h];
                    Dv = meta.rv[ti * rvs + 2 * h + 1];
                }
                const float bias = (lgl - lse2) * kLog2e;
                const int dq_row = valid ? (int)(((int64_t)b * sh.Hq + g * G + h) * T + t) : -1;
                // token r of the chunk, for its Gsum (read now: the metadata slot is
                // refilled once the chunk's last MMAs are issued)
                gs_slot = r < n ? meta.ent[r].z : -1;
                gs_tok = r < n ? meta.ent[r].x : 0;
                if (!tc::warp_wait_bar(&s_full[st], (uint32_t)((c >> 1) & 1), abort)) { fail = true; break; }
                tc::fence_after_sync();
                float rowsum = 0.f;
                uint32_t sv[32], pv[32];
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    tc::tmem_ld16(lane_base + (uint32_t)(st * 128 + hf * 32 + cb * 16), sv + cb * 16);
                    tc::tmem_ld16(lane_base + (uint32_t)(st * 128 + 64 + hf * 32 + cb * 16), pv + cb * 16);
                }
                tc::tmem_wait_ld();
                uint32_t pk[16], dk2[16];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const int kk = hf * 32 + k;
                    const float p0 = (kk <= kmax) ? exp2f(fmaf(__uint_as_float(sv[k]), qk, bias)) : 0.f;
                    const float p1 = (kk + 1 <= kmax) ? exp2f(fmaf(__uint_as_float(sv[k + 1]), qk, bias)) : 0.f;
                    const float d0 = p0 * (__uint_as_float(pv[k]) - Dv);
                    const float d1 = p1 * (__uint_as_float(pv[k + 1]) - Dv);
                    rowsum += d0 + d1;
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
                    pk[k / 2] = *reinterpret_cast<uint32_t*>(&hp);
                    dk2[k / 2] = *reinterpret_cast<uint32_t*>(&hd);
                }
                // P and dS of chunk c-1 must have been consumed by its MMAs before
                // they are overwritten; that also means the epilogue warps are done
                // with chunk c-2, whose row-id slot is reused here
                if (c >= 1 && !tc::warp_wait_bar(p_empty, (uint32_t)((c - 1) & 1), abort)) { fail = true; break; }
                if (hf == 0) {
                    ids[st * kRows + r] = dq_row;
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&ids_full[st]);
                }
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    const uint32_t off = tc::sw128_offset(r, hf * 32 + cb * 8);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + L::kP + off), "r"(pk[cb * 4]),
                                 "r"(pk[cb * 4 + 1]), "r"(pk[cb * 4 + 2]), "r"(pk[cb * 4 + 3])
                                 : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + L::kDS + off),
                                 "r"(dk2[cb * 4]), "r"(dk2[cb * 4 + 1]), "r"(dk2[cb * 4 + 2]), "r"(dk2[cb * 4 + 3])
                                 : "memory");
                }
                tc::fence_async_shared();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(p_full);
                // Gsum of the token: its G rows are in this chunk
                if (valid && !diag) atomicAdd(&gs[ti], rowsum);
            } while (false);
            // every P/dS warp takes this barrier once per chunk; it also tells them
            // all whether any of them (or another role) gave up on a wait, so that
            // they leave the loop together and no warp is left at a barrier
            if (tc::bar_red_or(1, 256, fail || *abort != 0)) break;
            if (hf == 0 && r < n) {
                if (gs_slot >= 0) a.gsum[((int64_t)bg * T + gs_tok) * K + gs_slot] = gs[r];
                gs[r] = 0.f;
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------- epilogue warps (0 - 3) ---
        const int r = warp * 32 + lane;            // chunk row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const float dscale = sh.scale;
        const int qd = lane & 3;
        bool ok = true;
        for (int c = 0; c < nc; ++c) {
            const int st = c & 1;
            if (!tc::warp_wait_bar(&ids_full[st], (uint32_t)((c >> 1) & 1), abort)) { ok = false; break; }
            const int dq_row = ids[st * kRows + r];
            // Lanes 4i..4i+3 trade 16-byte pieces (a 4x4 transpose) so that each
            // vector reduction of the warp covers 64 contiguous bytes of 8 rows:
            // whole 32-byte sectors reach L2 instead of halves.
            int rows4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) rows4[e] = __shfl_sync(0xffffffffu, dq_row, (lane & ~3) + e);
            if (!tc::warp_wait_bar(dq_full, (uint32_t)(c & 1), abort)) { ok = false; break; }
            tc::fence_after_sync();
#pragma unroll 1
            for (int cb = 0; cb < kD / 16; ++cb) {      // 16 columns at a time
                uint32_t v[16];
                tc::tmem_ld16(lane_base + kColDQ + cb * 16, v);
                tc::tmem_wait_ld();
                if (cb == kD / 16 - 1) {                 // dQ of this chunk is out of TMEM
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(dq_empty);
                }
                float x[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(v[e]) * dscale;
#pragma unroll
                for (int m = 1; m <= 2; m <<= 1) {
#pragma unroll
                    for (int k0 = 0; k0 < 4; ++k0) {
                        if (k0 & m) continue;
                        const int k1 = k0 | m;
                        const bool hi = (qd & m) != 0;
#pragma unroll
                        for (int f = 0; f < 4; ++f) {
                            const float snd = hi ? x[k0 * 4 + f] : x[k1 * 4 + f];
                            const float rcv = __shfl_xor_sync(0xffffffffu, snd, m);
                            if (hi) x[k0 * 4 + f] = rcv; else x[k1 * 4 + f] = rcv;
                        }
                    }
                }
                // x[4e .. 4e+3] = columns 4 qd .. 4 qd + 3 of this 16-column
                // slice, row (lane & ~3) + e
                const int col = cb * 16 + qd * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (rows4[e] >= 0)
                        tc::red_add_v4(a.dq_acc + (int64_t)rows4[e] * kD + col, x[4 * e], x[4 * e + 1],
                                       x[4 * e + 2], x[4 * e + 3]);
            }
        }
        // dV^T and dK^T: TMEM lane r holds column r of d for the block's 64 keys
        const int64_t kv0 = ((int64_t)bg * T + (int64_t)j * kBS) * kD;   // this group's block rows
        if (ok && tc::warp_wait_bar(done, 0u, abort)) {
            tc::fence_after_sync();
#pragma unroll 1
            for (int cb = 0; cb < kBS / 16; ++cb) {
                uint32_t vv[16], kv[16];
                tc::tmem_ld16(lane_base + kColDV + cb * 16, vv);
                tc::tmem_ld16(lane_base + kColDK + cb * 16, kv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int64_t at = kv0 + (int64_t)(cb * 16 + e) * kD + r;
                    const float fv = __uint_as_float(vv[e]), fk = __uint_as_float(kv[e]) * dscale;
                    if (a.dk32 != nullptr) {
                        a.dv32[at] = fv;
                        a.dk32[at] = fk;
                    } else {
                        a.dv[at] = __float2bfloat16_rn(fv);
                        a.dk[at] = __float2bfloat16_rn(fk);
                    }
                }
            }
        } else {
            // a wait gave up: the block's dK and dV are incomplete, mark them invalid
            const float nan = __int_as_float(0x7fc00000);
            for (int key = 0; key < kBS; ++key) {
                const int64_t at = kv0 + (int64_t)key * kD + r;
                if (a.dk32 != nullptr) {
                    a.dv32[at] = nan;
                    a.dk32[at] = nan;
                } else {
                    a.dv[at] = __float2bfloat16(nan);
                    a.dk[at] = __float2bfloat16(nan);
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 10) {
        // TMEM is released only after the last MMA that writes it
        if (lane == 0) tc::drain_wait(done, 0u);
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
    if (tid == 0 && *abort) atomicExch(a.aborted, 1);
}

}  // namespace

bool bwd_tc_supported(const Shape& s) {
    return s.dtype == SAS_DT_BF16 && s.D == kD && s.bs == kBS && s.K <= 64 && s.G <= 8 && s.q_offset == 0 &&
           s.T % kBS == 0 && s.nT <= 1024 && (int64_t)s.B * s.Hq * s.T < ((int64_t)1 << 31);
}

size_t bwd_tc_ws_bytes(const Shape& s) { return sel_stream_bytes(s, 2); }

cudaError_t launch_bwd_tc(const Shape& s, const void* q, const void* k, const void* v, const void* dO,
                          const float* lse, const float* Dd, const int32_t* idx, const float* gl,
                          const int32_t* nsel, const uint64_t* maskT, void* ws, float* dq_acc, void* dk, void* dv,
                          float* dk32, float* dv32, float* gsum, int* aborted, cudaStream_t st) {
    CUtensorMap mk, mv;
    if (!encode_bf16_2d(&mk, k, (uint64_t)s.B * s.Hkvp * s.T, kD, kBS) ||
        !encode_bf16_2d(&mv, v, (uint64_t)s.B * s.Hkvp * s.T, kD, kBS))
        return cudaErrorInvalidValue;
    BwdTcArgs a{};
    a.sh = s;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.dO = static_cast<const __nv_bfloat16*>(dO);
    a.ss = sel_stream_at(ws, s, 2);
    a.dq_acc = dq_acc;
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.dk32 = dk32;
    a.dv32 = dv32;
    a.gsum = gsum;
    a.aborted = aborted;
    a.tpc = kRows / s.G;
    a.meta_bytes = a.tpc * (16 + 4 * a.ss.rvs);
    // the streams carry each row's lse and D
    cudaError_t e = launch_sel_stream(s, maskT, idx, gl, nsel, lse, Dd, 2, a.ss, st);
    if (e != cudaSuccess) return e;
    const size_t smem = BwdSmem::total(a.meta_bytes) + 1024;
    e = cudaFuncSetAttribute(bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)s.B * s.Hkv * s.nT;
    {
        KernelTimer kt("bwd_tc", st);
        bwd_tc_kernel<<<(unsigned)grid, kThreads, smem, st>>>(mk, mv, a);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t set_bwd_tc_wait_limit(unsigned long long ns) {
    return cudaMemcpyToSymbol(g_sas_wait_limit_ns, &ns, sizeof(ns));
}

cudaError_t read_bwd_tc_timeouts(unsigned int* out) {
    return cudaMemcpyFromSymbol(out, g_sas_wait_timeouts, sizeof(unsigned int));
}

}  // namespace sas
