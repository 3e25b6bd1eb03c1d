// sparse_attn.cu -- KV-outer block-sparse attention, stage 1 of the two-stage forward
// ("MiniMax Sparse Attention" explainer, section 05-2).
//
// Each work item is one (group r, KV block b, chunk of the rows that selected b). Its K and V blocks
// are staged in shared memory once by TMA; the rows are processed in 128-row tensor-core tiles made
// of 128/G query positions x G heads ("query concatenation"), each position's G heads gathered by
// one TMA box from q[p, r*G .. r*G+G, :]. Per tile:
//   S = Q K^T                         tcgen05.mma, A = Q (smem), B = K (smem), D in TMEM
//   P = exp(S*scale - rowmax)         softmax warps, thread = TMEM lane = tile row; the causal mask
//                                     only applies to rows whose own block is b; P goes back to
//                                     TMEM as bf16 over the first 64 S columns
//   O = P V                           tcgen05.mma, A = P (TMEM), B = V (smem, MN-major)
//   partial[p, slot, h] = O / rowsum, lse = rowmax*scale + log(rowsum)
// A work item covers one KV block only, so no running-max rescaling is needed. Stage 2
// (combine.cu) merges the <= k partials of every (row, head) through their lse.
//
// Roles (512 threads, four warpgroups):
//   WG0: warp 0 = K/V TMA producer, warp 1 = S issuer + TMEM owner, warp 2 = tile scheduler and Q
//        gather (one TMA box per position, issued by the 32 lanes in parallel), warp 3 = PV issuer
//   WG1, WG2: softmax of even / odd tiles
//   WG3: epilogue of every tile (O / rowsum -> partial slot)
// Work items are claimed dynamically: the tile scheduler takes the next item of the launch's work
// list from a global atomic counter (so CTAs that drew short items take more), one item ahead of
// its own use, and hands it to the K/V producer through a 4-deep shared-memory item ring. It is the
// only role that reads the work list and the entries in global memory: it publishes every tile as
// a record (group, block, positions, their entries, item boundaries, the block's first token) in a
// shared-memory ring that the MMA issuers, the softmax and the epilogue consume, so none of them
// waits on a global load. The epilogue releases a record after its tile's PV. For a packed batch
// of sequences the block tables give each global block's first key row (K/V coordinates) and the
// query-row coordinate of its first token (the causal mask on the diagonal block).
// TMEM (512 columns): two 128-column S/P regions A[t % 2] at columns 0 and 128 (S, then P in
// columns 0-63) and two output regions O[t % 2] at columns 256 and 384. Two threads issue the
// MMAs, so neither's polling leaves the tensor pipe idle: the S issuer issues S(t) once PV(t-2)
// has consumed P(t-2) (region A[t % 2] free); the PV issuer issues PV(t) once P(t) is written and
// the epilogue of t-2 has read O[t % 2], which leaves the epilogue a full tile of slack.
// Barriers: s_full[2], p_full[2], pv_done[2] per S/P region; o_full[2], o_free[2] per O region;
// ml_full[4] hands each tile's row max and row sum from the softmax to the epilogue through shared
// memory (slot t % 4, rewritten by the softmax of t+4, which needs S(t+4), which needs PV(t+2),
// which needs the epilogue of t to have read O).
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace msa {

namespace {

template <int DH>
struct AttnCfg {
    static constexpr int NKC = DH / 64;          // 64-column (128-byte) chunks
    static constexpr int CHUNK = 128 * 128;      // bytes per chunk of a 128-row tile
    static constexpr int TILE = NKC * CHUNK;     // Q, K or V tile bytes
    static constexpr int NQ = 2;                 // Q stages
    static constexpr int SMEM = 1024 + NQ * TILE + 4 * TILE;
};

constexpr int kRing = 8; // tile records in flight between the scheduler and the epilogue

struct TileRec {
    int32_t r, b;  // GQA group, KV block
    int32_t npos;  // positions in the tile (1 .. 128/G); -1 marks the end of the CTA's work
    int32_t flags; // bit 0: first tile of its item, bit 1: last tile, bit 2: K/V stage of the item
    int32_t tok0;  // query-row coordinate of block b's first token (b * 128 for one sequence)
};

struct AttnShared {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t o_full[2], o_free[2];
    uint64_t ml_full[4];
    uint64_t tile_full[kRing], tile_free[kRing];
    uint64_t kvrec_full[4], kvrec_free[4];
    uint64_t done, done2;
    float2 ml[4][128]; // (row max of the raw scores, row sum of exp) per tile slot and row
    TileRec rec[kRing];
    msa_work_item kvrec[4]; // items handed to the K/V producer (len = 0: no more work)
    int32_t rec_e[kRing][128]; // entry (i*k + slot) of each position of the tile
    uint32_t tmem_base;
    int abort_flag;
};

constexpr uint32_t kNegInfBits = 0xff800000u;
constexpr int REG_LAUNCH = 128; // 65536 registers / 512 threads
constexpr int REG_PRODUCER = 56, REG_SOFTMAX = 184, REG_EPILOGUE = 88;
static_assert(REG_PRODUCER + 2 * REG_SOFTMAX + REG_EPILOGUE <= 4 * REG_LAUNCH, "register split exceeds the launch budget");

__device__ __forceinline__ uint32_t a_col(int t) { return (uint32_t)(t & 1) * 128; }
__device__ __forceinline__ uint32_t o_col(int t) { return 256u + (uint32_t)(t & 1) * 128; }

template <int DH, int G>
__global__ void __launch_bounds__(512, 1)
    sparse_attn_kernel(AttnArgs a, const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap)
{
    using C = AttnCfg<DH>;
    constexpr int PPT = 128 / G;
    constexpr int NQ = C::NQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                  // [NQ][TILE]
    uint8_t* sK = smem + NQ * C::TILE;   // [2][TILE]
    uint8_t* sV = sK + 2 * C::TILE;      // [2][TILE]
    AttnShared& sh = *reinterpret_cast<AttnShared*>(sV + 2 * C::TILE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    const int cta = blockIdx.x;
    const int64_t Nk = a.N * a.k;
    volatile int* abort_flag = &sh.abort_flag;
    const int j_base = a.window_items[a.w0];
    const int j_end = a.window_items[a.w1];
    const bool tl_on = a.timeline != nullptr && cta == 0;
#define TL(slot, tile)                                                                                    \
    do {                                                                                                  \
        if (tl_on && (tile) < a.timeline_tiles) a.timeline[(int64_t)(tile) * 16 + (slot)] = clock64();    \
    } while (0)

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.kv_full[i], 1);
            mbar_init(&sh.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.s_full[i], 1);
            mbar_init(&sh.p_full[i], 4);
            mbar_init(&sh.pv_done[i], 1);
            mbar_init(&sh.o_full[i], 1);
            mbar_init(&sh.o_free[i], 4);
        }
        for (int i = 0; i < NQ; ++i) {
            mbar_init(&sh.q_full[i], 1);
            mbar_init(&sh.q_empty[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&sh.ml_full[i], 4);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&sh.tile_full[i], 1);
            mbar_init(&sh.tile_free[i], 4);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&sh.kvrec_full[i], 1);
            mbar_init(&sh.kvrec_free[i], 1);
        }
        mbar_init(&sh.done, 1);
        mbar_init(&sh.done2, 1);
        sh.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (wg == 0) {
        reg_set<REG_PRODUCER, REG_LAUNCH>();
        if (warp == 0) {
            // -------------------------------------------------------- K/V producer
            if (lane == 0) {
                int it = 0;
                for (;; ++it) {
                    const int s4 = it & 3;
                    if (!wait_or_abort(&sh.kvrec_full[s4], (it >> 2) & 1, abort_flag, a.err, 38, kWaitLimit)) break;
                    const msa_work_item item = sh.kvrec[s4];
                    mbar_arrive(&sh.kvrec_free[s4]);
                    if (item.len <= 0) break;
                    const int s = it & 1;
                    if (!wait_or_abort(&sh.kv_empty[s], ((it >> 1) & 1) ^ 1, abort_flag, a.err, 20, kWaitLimit))
                        break;
                    const int tok0 = a.blk_tok ? a.blk_tok[item.b] : item.b * kBk;
                    mbar_arrive_expect_tx(&sh.kv_full[s], 2 * C::TILE);
                    for (int c = 0; c < C::NKC; ++c) {
                        tma_load_3d(sK + s * C::TILE + c * C::CHUNK, &kmap, &sh.kv_full[s], c * 64, item.r, tok0);
                        tma_load_3d(sV + s * C::TILE + c * C::CHUNK, &vmap, &sh.kv_full[s], c * 64, item.r, tok0);
                    }
                }
                for (int g = it - 1; g >= 0 && g >= it - 2; --g)
                    drain_wait(&sh.kv_full[g & 1], (g >> 1) & 1, a.err, 40, kWaitLimit);
            }
        } else if (warp == 2) {
            // -------------------------------------------------------- tile scheduler + Q gather
            // claim the next work item and hand it to the K/V producer (record slot n & 3)
            auto claim_and_publish = [&](int n, msa_work_item& item) -> bool {
                int j = 0;
                int w_ok = 1;
                if (lane == 0) {
                    j = j_base + atomicAdd(a.item_counter, 1);
                    item = j < j_end ? a.items[j] : msa_work_item{0, 0, 0, 0};
                    if (j < j_end && item.len <= 0) // the inversion never emits empty items: stop here
                        report_error(a.err, MSA_ERR_DEVICE_CHECK, 301);
                    if (n >= 4)
                        w_ok = wait_or_abort(&sh.kvrec_free[n & 3], ((n >> 2) & 1) ^ 1, abort_flag, a.err, 39,
                                             kWaitLimit);
                    if (w_ok) {
                        sh.kvrec[n & 3] = item;
                        mbar_arrive(&sh.kvrec_full[n & 3]);
                    }
                }
                item.r = __shfl_sync(0xffffffffu, item.r, 0);
                item.b = __shfl_sync(0xffffffffu, item.b, 0);
                item.start = __shfl_sync(0xffffffffu, item.start, 0);
                item.len = __shfl_sync(0xffffffffu, item.len, 0);
                return __shfl_sync(0xffffffffu, w_ok, 0) != 0;
            };
            int qt = 0, it = 0;
            msa_work_item item{0, 0, 0, 0};
            bool ok = claim_and_publish(0, item);
            while (ok && item.len > 0) {
                msa_work_item next{0, 0, 0, 0};
                ok = claim_and_publish(it + 1, next); // one item of look-ahead for the K/V producer
                if (!ok) break;
                const int32_t* ent = a.entries + (int64_t)item.r * Nk + item.start;
                const int ntiles = (item.len + PPT - 1) / PPT;
                // query-row coordinate of the block's first token (for the causal mask on the diagonal block)
                const int tok0 = a.blk_qtok ? a.blk_qtok[item.b] : a.blk_tok ? a.blk_tok[item.b] : item.b * kBk;
                for (int t = 0; t < ntiles; ++t, ++qt) {
                    const int qs = qt % NQ, rs = qt % kRing;
                    const int npos = min(PPT, item.len - t * PPT);
                    // fetch this tile's entries before waiting for anything
                    int e[(PPT + 31) / 32];
#pragma unroll
                    for (int u = 0; u < (PPT + 31) / 32; ++u) {
                        const int pl = lane + 32 * u;
                        e[u] = pl < npos ? ent[t * PPT + pl] : 0;
                    }
                    int w_ok = 1;
                    if (lane == 0 && qt >= kRing)
                        w_ok = wait_or_abort(&sh.tile_free[rs], ((qt / kRing) & 1) ^ 1, abort_flag, a.err, 33,
                                             kWaitLimit);
                    w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                    if (!w_ok) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int u = 0; u < (PPT + 31) / 32; ++u) {
                        const int pl = lane + 32 * u;
                        if (pl < npos) sh.rec_e[rs][pl] = e[u];
                    }
                    if (lane == 0)
                        sh.rec[rs] = TileRec{item.r, item.b, npos,
                                             (t == 0 ? 1 : 0) | (t == ntiles - 1 ? 2 : 0) | ((it & 1) << 2), tok0};
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.tile_full[rs]);
                    if (lane == 0)
                        w_ok = wait_or_abort(&sh.q_empty[qs], ((qt / NQ) & 1) ^ 1, abort_flag, a.err, 21, kWaitLimit);
                    w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                    if (!w_ok) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        TL(0, qt);
                        mbar_arrive_expect_tx(&sh.q_full[qs], npos * G * DH * 2);
                    }
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < (PPT + 31) / 32; ++u) {
                        const int pl = lane + 32 * u;
                        if (pl < npos) {
#pragma unroll
                            for (int c = 0; c < C::NKC; ++c)
                                tma_load_3d(sQ + qs * C::TILE + c * C::CHUNK + pl * G * 128, &qmap, &sh.q_full[qs],
                                            c * 64, item.r * G, e[u] / a.k);
                        }
                    }
                    if (lane == 0) TL(1, qt);
                }
                item = next;
                ++it;
            }
            const int n_tiles = qt;
            // two end records, so that each softmax warpgroup (even / odd tiles) meets one
            if (lane == 0 && ok) {
                for (int z = 0; z < 2; ++z, ++qt) {
                    const int rs = qt % kRing;
                    if (qt >= kRing && !wait_or_abort(&sh.tile_free[rs], ((qt / kRing) & 1) ^ 1, abort_flag, a.err,
                                                      33, kWaitLimit))
                        break;
                    sh.rec[rs] = TileRec{0, 0, -1, 0, 0};
                    mbar_arrive(&sh.tile_full[rs]);
                }
            }
            if (lane == 0)
                for (int g = n_tiles - 1; g >= 0 && g >= n_tiles - NQ; --g)
                    drain_wait(&sh.q_full[g % NQ], (g / NQ) & 1, a.err, 41, kWaitLimit);
        } else if (warp == 1) {
            // -------------------------------------------------------- S issuer: S(t) = Q K^T
            if (lane == 0) {
                constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
                const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
                int it = -1;
                uint64_t kdesc = 0;
                for (int qt = 0;; ++qt) {
                    const int rs = qt % kRing;
                    if (!poll_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 34, kWaitLimit)) break;
                    const TileRec rec = sh.rec[rs];
                    if (rec.npos < 0) break;
                    const int kvs = (rec.flags >> 2) & 1;
                    if (rec.flags & 1) {
                        ++it;
                        if (!poll_or_abort(&sh.kv_full[kvs], (it >> 1) & 1, abort_flag, a.err, 23, kWaitLimit)) break;
                        TL(8, qt);
                        kdesc = desc_kmajor(aK + kvs * C::TILE, 128);
                    }
                    const int qa = qt & 1, qs = qt % NQ;
                    // A[qt % 2] is free once PV(qt-2) has consumed P(qt-2)
                    if (!poll_or_abort(&sh.q_full[qs], (qt / NQ) & 1, abort_flag, a.err, 24, kWaitLimit) ||
                        (qt >= 2 && !poll_or_abort(&sh.pv_done[qa], ((qt >> 1) & 1) ^ 1, abort_flag, a.err, 25,
                                                   kWaitLimit)))
                        break;
                    TL(9, qt);
                    tc_fence_after();
                    const uint64_t qdesc = desc_kmajor(aQ + qs * C::TILE, 128);
                    const uint32_t sd = tmem + a_col(qt);
#pragma unroll
                    for (int ks = 0; ks < DH / 16; ++ks) {
                        const uint64_t off = (uint64_t)((((ks >> 2) * C::CHUNK) + (ks & 3) * 32) >> 4);
                        mma_ss(sd, qdesc + off, kdesc + off, idS, ks > 0);
                    }
                    tc_commit(&sh.s_full[qa]);
                    tc_commit(&sh.q_empty[qs]);
                    TL(2, qt);
                }
                tc_commit(&sh.done);
                drain_wait(&sh.done, 0, a.err, 42, kWaitLimit);
            }
        } else if (warp == 3) {
            // -------------------------------------------------------- PV issuer: O(t) = P(t) V
            if (lane == 0) {
                constexpr uint32_t idPV = idesc_bf16_f32(128, DH, true);
                const uint32_t aV = smem_u32(sV);
                int it = -1;
                uint64_t vdesc = 0;
                for (int qt = 0;; ++qt) {
                    const int rs = qt % kRing;
                    if (!poll_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 35, kWaitLimit)) break;
                    const TileRec rec = sh.rec[rs];
                    if (rec.npos < 0) break;
                    const int kvs = (rec.flags >> 2) & 1;
                    if (rec.flags & 1) {
                        ++it;
                        if (!poll_or_abort(&sh.kv_full[kvs], (it >> 1) & 1, abort_flag, a.err, 30, kWaitLimit)) break;
                        vdesc = smem_desc(aV + kvs * C::TILE, C::CHUNK, 1024, 128);
                    }
                    const int pa = qt & 1;
                    TL(10, qt);
                    // needs P(qt) and the epilogue of qt-2 to have read O[qt % 2]
                    if (!poll_or_abort(&sh.p_full[pa], (qt >> 1) & 1, abort_flag, a.err, 22, kWaitLimit) ||
                        (qt >= 2 && !poll_or_abort(&sh.o_free[pa], ((qt >> 1) & 1) ^ 1, abort_flag, a.err, 28,
                                                   kWaitLimit)))
                        break;
                    TL(12, qt);
                    tc_fence_after();
                    const uint32_t acol = tmem + a_col(qt);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) // 16 keys = 2048 bytes of V per step
                        mma_ts(tmem + o_col(qt), acol + ks * 8, vdesc + (uint64_t)(ks * 128), idPV, ks > 0);
                    tc_commit(&sh.pv_done[pa]);
                    tc_commit(&sh.o_full[pa]);
                    if (rec.flags & 2) tc_commit(&sh.kv_empty[kvs]);
                    TL(3, qt);
                }
                tc_commit(&sh.done2);
                drain_wait(&sh.done2, 0, a.err, 43, kWaitLimit);
            }
        }
    } else if (wg <= 2) {
        reg_set<REG_SOFTMAX, REG_LAUNCH>();
        // ------------------------------------------------------------ softmax
        const int beta = wg - 1;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int pl = row / G;
        const float sl2 = rsqrtf((float)DH) * 1.4426950408889634f;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        for (int qt = beta;; qt += 2) {
            const int rs = qt % kRing;
            if (!wait_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 36, kWaitLimit)) break;
            const TileRec rec = sh.rec[rs];
            if (rec.npos < 0) break;
            const int qa = qt & 1;
            const int limit = pl < rec.npos ? min(127, sh.rec_e[rs][pl] / a.k - rec.tok0) : 127;
            if (!wait_or_abort(&sh.s_full[qa], (qt >> 1) & 1, abort_flag, a.err, 26, kWaitLimit)) break;
            if (row == 0) TL(4, qt);
            tc_fence_after();
            const uint32_t sadr = lane_base + a_col(qt);
            uint32_t s[128];
            tmem_ld32_at<0>(sadr, s);
            tmem_ld32_at<32>(sadr + 32, s);
            tmem_ld32_at<64>(sadr + 64, s);
            tmem_ld32_at<96>(sadr + 96, s);
            tmem_ld_wait();
            if (row == 0) TL(14, qt);
            if (limit < 127) { // the query's own block: keys after the query are invisible
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > limit) s[c] = kNegInfBits;
            }
            float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
                m0 = max3f(m0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                m1 = max3f(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
            }
            const float m = fmaxf(m0, m1);
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            const uint64_t nmx2 = f2_pack(-m * sl2, -m * sl2);
            uint64_t l2 = 0;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t pk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c = c4 * 32 + 2 * q;
                    const uint64_t xx = f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2x2,
                                               nmx2);
                    const float e0 = ex2_approx(f2_lo(xx)), e1 = ex2_approx(f2_hi(xx));
                    l2 = f2_add(l2, f2_pack(e0, e1));
                    pk[q] = pack_bf16x2(e0, e1);
                }
                tmem_st16(sadr + c4 * 16, pk);
            }
            sh.ml[qt & 3][row] = make_float2(m, f2_lo(l2) + f2_hi(l2));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.p_full[qa]);
                mbar_arrive(&sh.ml_full[qt & 3]);
            }
            if (row == 0) TL(5, qt);
        }
    } else {
        reg_set<REG_EPILOGUE, REG_LAUNCH>();
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int pl = row / G, hh = row % G;
        const float scale = rsqrtf((float)DH);
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        for (int qt = 0;; ++qt) {
            if (row == 0) TL(15, qt);
            const int rs = qt % kRing;
            if (!wait_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 37, kWaitLimit)) break;
            const TileRec rec = sh.rec[rs];
            if (rec.npos < 0) break;
            const bool valid = pl < rec.npos;
            const int32_t e = valid ? sh.rec_e[rs][pl] : 0;
            const int p = e / a.k;
            const int slot = e - p * a.k;
            if (!wait_or_abort(&sh.o_full[qt & 1], (qt >> 1) & 1, abort_flag, a.err, 27, kWaitLimit) ||
                !wait_or_abort(&sh.ml_full[qt & 3], (qt >> 2) & 1, abort_flag, a.err, 29, kWaitLimit))
                break;
            if (row == 0) TL(6, qt);
            tc_fence_after();
            const float2 ml = sh.ml[qt & 3][row];
            const float inv_l = 1.f / ml.y;
            const int h = rec.r * G + hh;
            const int64_t prow = (int64_t)(p - a.row0);
            bool store = valid;
            if (valid && (prow < 0 || prow >= a.rows_pass || slot < 0 || slot >= a.k)) {
                report_error(a.err, MSA_ERR_DEVICE_CHECK, 300); // entry outside this pass: skip it
                store = false;
            }
            // partial layout [row][slot][d_h/8][H_q][8]: the G heads of a position are adjacent
            // 16-byte units, so each warp-wide store writes contiguous runs
            uint4* d4 = reinterpret_cast<uint4*>(a.o_part + (prow * a.k + slot) * (int64_t)a.H_q * DH) + h;
            const uint64_t il2 = f2_pack(inv_l, inv_l);
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_base + o_col(qt) + c * 32, o);
                tmem_ld_wait();
                if (c == DH / 32 - 1) { // O fully read: PV of the next tile may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&sh.o_free[qt & 1]);
                        mbar_arrive(&sh.tile_free[rs]); // S, softmax and PV of qt are done with the record
                    }
                    if (row == 0) TL(13, qt);
                }
                if (store) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            const uint64_t y = f2_mul(
                                f2_pack(__uint_as_float(o[8 * q + 2 * z]), __uint_as_float(o[8 * q + 2 * z + 1])),
                                il2);
                            w[z] = pack_bf16x2(f2_lo(y), f2_hi(y));
                        }
                        d4[(c * 4 + q) * a.H_q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (store) a.lse_part[(prow * a.k + slot) * a.H_q + h] = ml.x * scale + logf(ml.y);
            if (row == 0) TL(7, qt);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
#undef TL
}

template <int DH, int G>
cudaError_t launch_cfg(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t s, int n_sm)
{
    using C = AttnCfg<DH>;
    const int smem = C::SMEM + (int)sizeof(AttnShared);
    static_assert(AttnCfg<DH>::SMEM + sizeof(AttnShared) <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<DH, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    sparse_attn_kernel<DH, G><<<n_sm, 512, smem, s>>>(a, qmap, kmap, vmap);
    note_launch(1);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_dh(const AttnArgs& a, int G, const CUtensorMap& qmap, const CUtensorMap& kmap,
                      const CUtensorMap& vmap, cudaStream_t s, int n_sm)
{
    switch (G) {
    case 1: return launch_cfg<DH, 1>(a, qmap, kmap, vmap, s, n_sm);
    case 2: return launch_cfg<DH, 2>(a, qmap, kmap, vmap, s, n_sm);
    case 4: return launch_cfg<DH, 4>(a, qmap, kmap, vmap, s, n_sm);
    case 8: return launch_cfg<DH, 8>(a, qmap, kmap, vmap, s, n_sm);
    case 16: return launch_cfg<DH, 16>(a, qmap, kmap, vmap, s, n_sm);
    case 32: return launch_cfg<DH, 32>(a, qmap, kmap, vmap, s, n_sm);
    case 64: return launch_cfg<DH, 64>(a, qmap, kmap, vmap, s, n_sm);
    case 128: return launch_cfg<DH, 128>(a, qmap, kmap, vmap, s, n_sm);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace

cudaError_t launch_sparse_attn(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                               const CUtensorMap& vmap, cudaStream_t s)
{
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int G = a.H_q / a.H_kv;
    if (a.d_h == 64) return launch_dh<64>(a, G, qmap, kmap, vmap, s, n_sm);
    if (a.d_h == 128) return launch_dh<128>(a, G, qmap, kmap, vmap, s, n_sm);
    return cudaErrorInvalidValue;
}

} // namespace msa
