// sparse_attn.cu -- KV-outer block-sparse attention, stage 1 of the two-stage forward
// ("MiniMax Sparse Attention" explainer, section 05-2).
//
// Each work item is one (group r, KV block b, chunk of the rows that selected b). Its K and V blocks
// are staged in shared memory once by TMA; the rows are processed in 128-row tensor-core tiles made
// of 128/G query positions x G heads ("query concatenation"), each position's G heads gathered by
// TMA from q[p, r*G .. r*G+G, :] (one box per position when G >= 8). Per tile:
//   S = Q K^T                         tcgen05.mma, A = Q (smem), B = K (smem), D in TMEM
//   P = exp(S*scale - rowmax)         softmax warps, thread = TMEM lane = tile row; the causal mask
//                                     only applies to rows whose own block is b; P goes back to
//                                     TMEM as bf16 over the first 64 S columns
//   partial[p, slot, h] = O / rowsum(bf16 P), lse = rowmax*scale + log(rowsum(P))
//   O = P V                           tcgen05.mma, A = P (TMEM), B = V (smem, MN-major)
// A work item covers one KV block only, so no running-max rescaling is needed. Stage 2
// (combine.cu) merges the <= k partials of every (row, head) through their lse.
//
// Roles (512 threads, four warpgroups):
//   WG0: warp 0 = K/V TMA producer, warp 1 = S issuer + TMEM owner, warp 2 = tile scheduler and Q
//        gather (TMA boxes issued by the 32 lanes in parallel), warp 3 = PV issuer
//   WG1, WG2: softmax, one 64-column half of every tile each
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
//
// Pipeline depth. A tile's S/P columns stay busy from S through the softmax until PV has read P,
// while its output columns are busy only from PV until the epilogue has read them, so TMEM (512
// columns) holds three S/P regions R[t % 3] at columns 0, 128, 256 (S, then P in the first 64
// columns) and one output region at columns 384-511: three tiles are in flight between S and PV.
// Both softmax warpgroups work on every tile (one 64-column half of the keys each, exchanging the
// row maxima through shared memory), which halves a tile's softmax latency.
// Two threads issue the MMAs. A thread stays busy about as long as the tensor pipe takes to run
// what it issues, and every barrier wait or tcgen05.commit costs it tens of cycles, so each issuer
// reads only the first record of an item (which carries the item's tile count) and per tile waits
// on two barriers and commits one: the S issuer waits for Q(t) and for PV(t-3) (region R[t % 3]
// free) and commits s_full, which also frees Q stage t % 3; the PV issuer waits for P(t) and for the
// epilogue's read of O(t-1) and commits pv_done, which frees region R[t % 3] and hands O(t) to the
// epilogue. Q has three shared-memory stages (stage t % 3, refilled for t+3 once S(t) completed).
// K and V of consecutive items rotate through three 128-row buffers in load order K0 V0 K1 V1 ...:
// load n goes to buffer n % 3 once load n-3 is released (the K of an item after its last S, its V
// after its last PV), so the next item's K and V stream in while the current item's tiles run.
// The softmax hands each tile's row max and row sums to the epilogue through shared memory (slot
// t % 4, ml_full[t % 4]; rewritten by the softmax of t+4, which needs S(t+4), which needs PV(t+1),
// which needs the epilogue of t to have read O(t), after it read the slot).
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace msa {

namespace {

template <int DH, int G, bool F8>
struct AttnCfg {
    static constexpr int EB = F8 ? 1 : 2;        // bytes per operand element (E4M3 or bf16)
    static constexpr int NKC = DH * EB / 128;    // 128-byte chunks of an operand row
    static constexpr int CE = 128 / EB;          // elements per chunk
    static constexpr int KSTEPS = DH * EB / 32;  // S MMAs per tile (32 bytes of K each)
    static constexpr int CHUNK = 128 * 128;      // bytes per chunk of a 128-row tile
    static constexpr int TILE = NKC * CHUNK;     // Q, K or V tile bytes
    static constexpr int NQ = 3;                 // Q stages
    static constexpr int NKV = 3;                // K/V buffers
    static constexpr int SMEM = 1024 + (NQ + NKV) * TILE;
    // Q tile layout. G >= 8: position-major, one TMA box per position laid out as
    // [head group of 8][chunk][8 heads][128 B]: 8-row group g = p * G/8 + hg sits at g * QSBO and
    // chunk c at + c * 1024. G < 8: chunk-major like K ([chunk][row][128 B]), one box per
    // (position, chunk).
    static constexpr bool QPOS = G >= 8;
    static constexpr int QSBO = QPOS ? NKC * 1024 : 1024; // bytes between 8-row groups
    static constexpr int QCHUNK = QPOS ? 1024 : CHUNK;    // bytes between 128-byte chunks
};

constexpr int kRing = 8;    // tile records in flight between the scheduler and the epilogue
constexpr int kRegions = 3; // S/P regions in TMEM
constexpr uint32_t kOCol = 384;

struct TileRec {
    int32_t r, b;   // GQA group, KV block
    int32_t npos;   // positions in the tile (1 .. 128/G); -1 marks the end of the CTA's work
    int32_t flags;  // bit 0: first tile of its item, bit 1: last tile
    int32_t tok0;   // query-row coordinate of block b's first token (b * 128 for one sequence)
    int32_t ntiles; // tiles of the item (the MMA issuers read only each item's first record)
    int32_t item;   // the CTA's item counter (K of item i is load 2i, V load 2i+1, buffer = load % 3)
};

struct AttnShared {
    uint64_t kv_full[3], kv_empty[3];
    uint64_t q_full[3];
    uint64_t s_full[kRegions], p_full[kRegions], pv_done[kRegions];
    uint64_t o_free;
    uint64_t ml_full[4];
    uint64_t tile_full[kRing], tile_free[kRing];
    uint64_t kvrec_full[4], kvrec_free[4];
    uint64_t done, done2;
    uint64_t xbar[2][4];    // [tile & 1][lane quarter]: both softmax warps of the quarter hold their max
    float xmax[2][2][128];  // [tile & 1][column half][row]: the halves' row maxima, exchanged
    float mrow[4][128];     // [tile slot][row]: row max of the raw scores
    float2 lsum[4][2][128]; // [tile slot][column half][row]: (sum of exp, sum of the bf16-rounded P)
    TileRec rec[kRing];
    msa_work_item kvrec[4]; // items handed to the K/V producer (len = 0: no more work)
    int32_t rec_e[kRing][128]; // entry (i*k + slot) of each position of the tile
    // FP8 only: per K/V buffer holding a V load, the item's k scales, v scales and their reciprocals
    // (128 tokens each, loaded with V: the slot lives until the item's last PV) and 448 / (largest
    // v scale of the block)
    alignas(16) float fscl[3][3][128];
    float fcb[3];
    uint32_t tmem_base;
    int abort_flag;
};

constexpr uint32_t kNegInfBits = 0xff800000u;
constexpr int REG_LAUNCH = 128; // 65536 registers / 512 threads
constexpr int REG_PRODUCER = 80, REG_SOFTMAX = 128, REG_EPILOGUE = 176;
static_assert(REG_PRODUCER + 2 * REG_SOFTMAX + REG_EPILOGUE <= 4 * REG_LAUNCH, "register split exceeds the launch budget");

__device__ __forceinline__ uint32_t a_col(int t) { return (uint32_t)(t % kRegions) * 128; }

template <int DH, int G, bool F8>
__global__ void __launch_bounds__(512, 1)
    sparse_attn_kernel(AttnArgs a, const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap)
{
    using C = AttnCfg<DH, G, F8>;
    constexpr int PPT = 128 / G;
    constexpr int NQ = C::NQ, NKV = C::NKV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                  // [NQ][TILE]
    uint8_t* sKV = smem + NQ * C::TILE;  // [NKV][TILE]
    AttnShared& sh = *reinterpret_cast<AttnShared*>(sKV + NKV * C::TILE);

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
        if (tl_on && (tile) < a.timeline_tiles) a.timeline[(int64_t)(tile) * 48 + (slot)] = clock64();    \
    } while (0)

    if (threadIdx.x == 0) {
        for (int i = 0; i < NKV; ++i) {
            mbar_init(&sh.kv_full[i], 1);
            mbar_init(&sh.kv_empty[i], 1);
        }
        for (int i = 0; i < kRegions; ++i) {
            mbar_init(&sh.s_full[i], 1);
            mbar_init(&sh.p_full[i], 8);
            mbar_init(&sh.pv_done[i], 1);
        }
        mbar_init(&sh.o_free, 4);
        for (int i = 0; i < NQ; ++i) mbar_init(&sh.q_full[i], 1);
        for (int i = 0; i < 4; ++i) mbar_init(&sh.ml_full[i], 8);
        for (int i = 0; i < 8; ++i) mbar_init(&sh.xbar[i >> 2][i & 3], 2);
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
            // loads n = 2i (K of item i) and 2i+1 (V of item i) go to buffer n % 3
            if (lane == 0) {
                int n = 0;
                bool ok = true;
                for (int it = 0; ok; ++it) {
                    const int s4 = it & 3;
                    if (!wait_or_abort(&sh.kvrec_full[s4], (it >> 2) & 1, abort_flag, a.err, 38, kWaitLimit)) break;
                    const msa_work_item item = sh.kvrec[s4];
                    mbar_arrive(&sh.kvrec_free[s4]);
                    if (item.len <= 0) break;
                    const int tok0 = a.blk_tok ? a.blk_tok[item.b] : item.b * kBk;
                    for (int kv = 0; kv < 2; ++kv, ++n) {
                        const int buf = n % NKV;
                        if (!wait_or_abort(&sh.kv_empty[buf], ((n / NKV) & 1) ^ 1, abort_flag, a.err, 20,
                                           kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        if constexpr (F8) {
                            if (kv) { // with V: the item's k, v, 1/v scales (512 B each) and 448 / block max
                                const float vmax = a.vblkmax[(int64_t)item.r * a.nb + item.b];
                                sh.fcb[buf] = vmax > 0.f ? 448.f / vmax : 1.f;
                                mbar_arrive_expect_tx(&sh.kv_full[buf], C::TILE + 3 * 512);
                                const int64_t so = (int64_t)item.r * a.sstride + tok0;
                                bulk_load(sh.fscl[buf][0], a.ks + so, 512, &sh.kv_full[buf]);
                                bulk_load(sh.fscl[buf][1], a.vs + so, 512, &sh.kv_full[buf]);
                                bulk_load(sh.fscl[buf][2], a.rvs + so, 512, &sh.kv_full[buf]);
                            } else {
                                mbar_arrive_expect_tx(&sh.kv_full[buf], C::TILE);
                            }
                        } else {
                            mbar_arrive_expect_tx(&sh.kv_full[buf], C::TILE);
                        }
                        for (int c = 0; c < C::NKC; ++c)
                            tma_load_3d(sKV + buf * C::TILE + c * C::CHUNK, kv ? &vmap : &kmap, &sh.kv_full[buf],
                                        c * C::CE, item.r, tok0);
                    }
                }
                for (int g = n - 1; g >= 0 && g >= n - NKV; --g)
                    drain_wait(&sh.kv_full[g % NKV], (g / NKV) & 1, a.err, 40, kWaitLimit);
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
                        sh.rec[rs] = TileRec{item.r, item.b, npos, (t == 0 ? 1 : 0) | (t == ntiles - 1 ? 2 : 0), tok0,
                                             ntiles, it};
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.tile_full[rs]);
                    // Q stage qs is free once S(qt-3), the last reader of the stage, has completed
                    if (lane == 0)
                        w_ok = wait_or_abort(&sh.s_full[qs], ((qt / NQ) & 1) ^ 1, abort_flag, a.err, 21, kWaitLimit);
                    w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                    if (!w_ok) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        TL(0, qt);
                        mbar_arrive_expect_tx(&sh.q_full[qs], npos * G * DH * C::EB);
                    }
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < (PPT + 31) / 32; ++u) {
                        const int pl = lane + 32 * u;
                        if (pl < npos) {
                            uint8_t* dst = sQ + qs * C::TILE;
                            if constexpr (C::QPOS) {
                                tma_load_5d(dst + pl * (G * DH * C::EB), &qmap, &sh.q_full[qs], 0, 0, 0,
                                            item.r * (G / 8), e[u] / a.k);
                            } else {
#pragma unroll
                                for (int c = 0; c < C::NKC; ++c)
                                    tma_load_3d(dst + c * C::CHUNK + pl * G * 128, &qmap, &sh.q_full[qs], c * C::CE,
                                                item.r * G, e[u] / a.k);
                            }
                        }
                    }
                    if (lane == 0) TL(1, qt);
                }
                item = next;
                ++it;
            }
            const int n_tiles = qt;
            // the end record, read by every consumer role
            if (lane == 0 && ok) {
                const int rs = qt % kRing;
                if (qt < kRing ||
                    wait_or_abort(&sh.tile_free[rs], ((qt / kRing) & 1) ^ 1, abort_flag, a.err, 33, kWaitLimit)) {
                    sh.rec[rs] = TileRec{0, 0, -1, 0, 0, 0, 0};
                    mbar_arrive(&sh.tile_full[rs]);
                }
            }
            if (lane == 0)
                for (int g = n_tiles - 1; g >= 0 && g >= n_tiles - NQ; --g)
                    drain_wait(&sh.q_full[g % NQ], (g / NQ) & 1, a.err, 41, kWaitLimit);
        } else if (warp == 1) {
            // -------------------------------------------------------- S issuer: S(t) = Q K^T
            // reads only each item's first record; per tile it waits for Q(t) and for PV(t-3) to have
            // consumed P(t-3) (region R[t % 3] free), and commits one barrier (s_full, which also
            // frees Q stage t % 3 for the scheduler)
            if (lane == 0) {
                constexpr uint32_t idS = F8 ? idesc_e4m3_f32(128, 128, false) : idesc_bf16_f32(128, 128, false);
                const uint32_t aQ = smem_u32(sQ), aKV = smem_u32(sKV);
                int qt = 0;
                bool ok = true;
                for (int it = 0; ok; ++it) {
                    const int rs = qt % kRing;
                    if (!wait_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 34, kWaitLimit)) break;
                    const TileRec rec = sh.rec[rs];
                    if (rec.npos < 0) break;
                    const int kb = (2 * it) % NKV; // K of item it = load 2*it
                    if (!wait_or_abort(&sh.kv_full[kb], ((2 * it) / NKV) & 1, abort_flag, a.err, 23, kWaitLimit)) break;
                    const uint64_t kdesc = desc_kmajor(aKV + kb * C::TILE, 128);
                    TL(8, qt);
                    for (int t = 0; t < rec.ntiles; ++t, ++qt) {
                        const int reg = qt % kRegions;
                        if (!wait_or_abort(&sh.q_full[reg], (qt / NQ) & 1, abort_flag, a.err, 24, kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        TL(38, qt);
                        if (!wait_or_abort(&sh.pv_done[reg], ((qt / kRegions) & 1) ^ 1, abort_flag, a.err, 25,
                                           kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        TL(9, qt);
                        tc_fence_after();
                        const uint64_t qdesc = smem_desc(aQ + reg * C::TILE, 16, C::QSBO, 128);
                        const uint32_t sd = tmem + a_col(qt);
#pragma unroll
                        for (int ks = 0; ks < C::KSTEPS; ++ks) {
                            const uint64_t qoff = (uint64_t)((((ks >> 2) * C::QCHUNK) + (ks & 3) * 32) >> 4);
                            const uint64_t koff = (uint64_t)((((ks >> 2) * C::CHUNK) + (ks & 3) * 32) >> 4);
                            if constexpr (F8)
                                mma_ss_f8(sd, qdesc + qoff, kdesc + koff, idS, ks > 0);
                            else
                                mma_ss(sd, qdesc + qoff, kdesc + koff, idS, ks > 0);
                        }
                        TL(32, qt);
                        tc_commit(&sh.s_full[reg]);
                        if (t == rec.ntiles - 1) tc_commit(&sh.kv_empty[kb]); // the item's K is no longer read
                        TL(2, qt);
                    }
                }
                tc_commit(&sh.done);
                drain_wait(&sh.done, 0, a.err, 42, kWaitLimit);
            }
        } else if (warp == 3) {
            // -------------------------------------------------------- PV issuer: O(t) = P(t) V
            // reads only each item's first record; per tile it waits for P(t) and for the epilogue's
            // read of O(t-1), and commits one barrier (pv_done: region R[t % 3] free, O(t) ready)
            if (lane == 0) {
                constexpr uint32_t idPV = F8 ? idesc_e4m3_f32(128, DH, true) : idesc_bf16_f32(128, DH, true);
                const uint32_t aKV = smem_u32(sKV);
                int qt = 0;
                bool ok = true;
                for (int it = 0; ok; ++it) {
                    const int rs = qt % kRing;
                    if (!wait_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 35, kWaitLimit)) break;
                    const TileRec rec = sh.rec[rs];
                    if (rec.npos < 0) break;
                    const int vb = (2 * it + 1) % NKV; // V of item it = load 2*it + 1
                    if (!wait_or_abort(&sh.kv_full[vb], ((2 * it + 1) / NKV) & 1, abort_flag, a.err, 30, kWaitLimit))
                        break;
                    const uint64_t vdesc = smem_desc(aKV + vb * C::TILE, C::CHUNK, 1024, 128);
                    for (int t = 0; t < rec.ntiles; ++t, ++qt) {
                        const int reg = qt % kRegions;
                        if (!wait_or_abort(&sh.p_full[reg], (qt / kRegions) & 1, abort_flag, a.err, 22, kWaitLimit) ||
                            !wait_or_abort(&sh.o_free, (qt & 1) ^ 1, abort_flag, a.err, 28, kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        TL(12, qt);
                        tc_fence_after();
                        const uint32_t acol = tmem + a_col(qt);
                        // one step = 32 bytes of keys: 16 (bf16) or 32 (E4M3) rows of V, 8 columns of P
#pragma unroll
                        for (int ks = 0; ks < 128 * C::EB / 32; ++ks) {
                            if constexpr (F8)
                                mma_ts_f8(tmem + kOCol, acol + ks * 8, vdesc + (uint64_t)(ks * 32 * DH / 16), idPV,
                                          ks > 0);
                            else
                                mma_ts(tmem + kOCol, acol + ks * 8, vdesc + (uint64_t)(ks * 128), idPV, ks > 0);
                        }
                        TL(36, qt);
                        tc_commit(&sh.pv_done[reg]);
                        if (t == rec.ntiles - 1) tc_commit(&sh.kv_empty[vb]); // the item's V is no longer read
                        TL(3, qt);
                    }
                }
                tc_commit(&sh.done2);
                drain_wait(&sh.done2, 0, a.err, 43, kWaitLimit);
            }
        }
    } else if (wg <= 2) {
        reg_set<REG_SOFTMAX, REG_LAUNCH>();
        // ------------------------------------------------------------ softmax
        // Both warpgroups work on every tile: warpgroup beta takes key columns 64*beta .. +63 of the
        // rows of its TMEM lane quarter. The two warps of a lane quarter exchange their row maxima
        // through shared memory (an mbarrier per tile parity and quarter, two arrivals), then each
        // writes its half of P.
        const int beta = wg - 1;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int pl = row / G;
        const float sl2 = rsqrtf((float)DH) * 1.4426950408889634f;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        for (int qt = 0;; ++qt) {
            const int rs = qt % kRing;
            if (!wait_or_abort(&sh.tile_full[rs], (qt / kRing) & 1, abort_flag, a.err, 36, kWaitLimit)) break;
            const TileRec rec = sh.rec[rs];
            if (rec.npos < 0) break;
            const int reg = qt % kRegions;
            const int e_row = pl < rec.npos ? sh.rec_e[rs][pl] : 0;
            // last visible key column of this half (keys after the query are masked on the diagonal block)
            const int limit = (pl < rec.npos ? min(127, e_row / a.k - rec.tok0) : 127) - 64 * beta;
            float sq = 1.f; // FP8: the row's q scale
            if constexpr (F8) {
                if (pl < rec.npos) sq = a.qs[(int64_t)(rec.r * G + row % G) * a.sstride + e_row / a.k];
            }
            if (!wait_or_abort(&sh.s_full[reg], (qt / kRegions) & 1, abort_flag, a.err, 26, kWaitLimit)) break;
            if (row == 0 && beta == 0) TL(4, qt);
            tc_fence_after();
            const uint32_t sadr = lane_base + a_col(qt);
            uint32_t s[64];
            tmem_ld32_at<0>(sadr + 64 * beta, s);
            tmem_ld32_at<32>(sadr + 64 * beta + 32, s);
            tmem_ld_wait();
            if (row == 0 && beta == 0) TL(14, qt);
            const int vbuf = (2 * rec.item + 1) % NKV; // FP8: the buffer of the item's V load and scales
            if constexpr (F8) {
                // logits in units of the codes: q8 . k8 * s_k (the row's s_q * scale enters the exponent)
                if (!wait_or_abort(&sh.kv_full[vbuf], ((2 * rec.item + 1) / NKV) & 1, abort_flag, a.err, 45,
                                   kWaitLimit))
                    break;
                const float4* ksc = reinterpret_cast<const float4*>(sh.fscl[vbuf][0] + 64 * beta);
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 k4 = ksc[c / 4];
                    s[c] = __float_as_uint(__uint_as_float(s[c]) * k4.x);
                    s[c + 1] = __float_as_uint(__uint_as_float(s[c + 1]) * k4.y);
                    s[c + 2] = __float_as_uint(__uint_as_float(s[c + 2]) * k4.z);
                    s[c + 3] = __float_as_uint(__uint_as_float(s[c + 3]) * k4.w);
                }
            }
            if (limit < 63) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c > limit) s[c] = kNegInfBits;
            }
            float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                m0 = max3f(m0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                m1 = max3f(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
            }
            sh.xmax[qt & 1][beta][row] = fmaxf(m0, m1);
            // both halves of S are in registers before either half's P overwrites TMEM columns 0-63
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.xbar[qt & 1][quarter]);
            if (!wait_or_abort(&sh.xbar[qt & 1][quarter], (qt >> 1) & 1, abort_flag, a.err, 44, kWaitLimit)) break;
            tc_fence_after();
            if (row == 0 && beta == 0) TL(33, qt);
            const float m = fmaxf(sh.xmax[qt & 1][0][row], sh.xmax[qt & 1][1][row]);
            const float cl2 = F8 ? sl2 * sq : sl2; // logit -> log2 units
            const uint64_t sl2x2 = f2_pack(cl2, cl2);
            const uint64_t nmx2 = f2_pack(-m * cl2, -m * cl2);
            uint64_t l2 = 0, lr2 = 0;
            if constexpr (F8) {
                // P' = P * s_v * C_b (at most 448) rounded to E4M3 for the PV product; the row sum of the
                // weights it stands for, P'_q / (s_v * C_b) = P'_q * (1 / s_v) / C_b, normalises O: the
                // partial is O / sum(P'_q / s_v) (the C_b cancel), an exact weighted average of V rows
                const float cb = sh.fcb[vbuf];
                const float4* vsc = reinterpret_cast<const float4*>(sh.fscl[vbuf][1] + 64 * beta);
                const float4* rvc = reinterpret_cast<const float4*>(sh.fscl[vbuf][2] + 64 * beta);
                uint32_t pk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c = 4 * q;
                    const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2x2, nmx2);
                    const uint64_t x23 =
                        f2_fma(f2_pack(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), sl2x2, nmx2);
                    const float e0 = ex2_approx(f2_lo(x01)), e1 = ex2_approx(f2_hi(x01));
                    const float e2 = ex2_approx(f2_lo(x23)), e3 = ex2_approx(f2_hi(x23));
                    l2 = f2_add(l2, f2_add(f2_pack(e0, e1), f2_pack(e2, e3)));
                    const float4 v4 = vsc[q], r4 = rvc[q];
                    const uint32_t w01 = e4m3x2_pack(e0 * v4.x * cb, e1 * v4.y * cb);
                    const uint32_t w23 = e4m3x2_pack(e2 * v4.z * cb, e3 * v4.w * cb);
                    pk[q] = w01 | (w23 << 16);
                    const float2 d01 = e4m3x2_unpack(w01), d23 = e4m3x2_unpack(w23);
                    lr2 = f2_fma(f2_pack(d01.x, d01.y), f2_pack(r4.x, r4.y), lr2);
                    lr2 = f2_fma(f2_pack(d23.x, d23.y), f2_pack(r4.z, r4.w), lr2);
                }
                tmem_st16(sadr + 16 * beta, pk);
            } else {
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
                uint32_t pk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c = c4 * 32 + 2 * q;
                    const uint64_t xx = f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2x2,
                                               nmx2);
                    const float e0 = ex2_approx(f2_lo(xx)), e1 = ex2_approx(f2_hi(xx));
                    pk[q] = pack_bf16x2(e0, e1);
                    l2 = f2_add(l2, f2_pack(e0, e1));
                    lr2 = f2_add(lr2, f2_pack(bf16_lo(pk[q]), bf16_hi(pk[q])));
                }
                tmem_st16(sadr + 32 * beta + c4 * 16, pk);
            }
            }
            // the exact sum gives the lse (the combine's merge weight); the sum of the bf16-rounded P
            // that the PV product uses normalises O, so each partial is an exact weighted average
            sh.lsum[qt & 3][beta][row] = make_float2(f2_lo(l2) + f2_hi(l2), f2_lo(lr2) + f2_hi(lr2));
            // row max: of the raw scores (bf16), of the logits in natural units (FP8)
            if (beta == 0) sh.mrow[qt & 3][row] = F8 ? m * sq * (sl2 * 0.6931471805599453f) : m;
            if (row == 0 && beta == 0) TL(34, qt);
            tmem_st_wait();
            if (row == 0 && beta == 0) TL(35, qt);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.p_full[reg]);
                mbar_arrive(&sh.ml_full[qt & 3]);
                TL(16 + 4 * beta + quarter, qt);
            }
            if (row == 0 && beta == 0) TL(5, qt);
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
            if (!wait_or_abort(&sh.pv_done[qt % kRegions], (qt / kRegions) & 1, abort_flag, a.err, 27, kWaitLimit) ||
                !wait_or_abort(&sh.ml_full[qt & 3], (qt >> 2) & 1, abort_flag, a.err, 29, kWaitLimit))
                break;
            if (row == 0) TL(6, qt);
            tc_fence_after();
            const float2 la = sh.lsum[qt & 3][0][row], lb = sh.lsum[qt & 3][1][row];
            const float lse_row = (F8 ? sh.mrow[qt & 3][row] : sh.mrow[qt & 3][row] * scale) + logf(la.x + lb.x);
            const float inv_l = 1.f / (la.y + lb.y);
            const int h = rec.r * G + hh;
            const int64_t prow = (int64_t)(p - a.row0);
            bool store = valid;
            if (valid && (prow < 0 || prow >= a.rows_pass || slot < 0 || slot >= a.k)) {
                report_error(a.err, MSA_ERR_DEVICE_CHECK, 300); // entry outside this pass: skip it
                store = false;
            }
            // partial layout [row][slot][d_h/16][H_q][16]: the G heads of a position are adjacent
            // 32-byte units, so each warp-wide 32-byte store writes contiguous runs (half as many store
            // instructions as 16-byte units would take for the same bytes)
            uint32_t* d8 = reinterpret_cast<uint32_t*>(a.o_part + (prow * a.k + slot) * (int64_t)a.H_q * DH) + h * 8;
            const uint64_t il2 = f2_pack(inv_l, inv_l);
            // the whole output row is read with one wait and the region released to the next PV before
            // any conversion; the bf16 pairs are then packed in place (word z from words 2z, 2z+1)
            uint32_t w[DH];
            tmem_ld32_at<0>(lane_base + kOCol, w);
            tmem_ld32_at<32>(lane_base + kOCol + 32, w);
            if constexpr (DH > 64) {
                tmem_ld32_at<64>(lane_base + kOCol + 64, w);
                tmem_ld32_at<96>(lane_base + kOCol + 96, w);
            }
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.o_free);
                mbar_arrive(&sh.tile_free[rs]); // S, softmax and PV of qt are done with the record
                TL(24 + quarter, qt);
            }
            if (row == 0) TL(13, qt);
#pragma unroll
            for (int z = 0; z < DH / 2; ++z) {
                const uint64_t y = f2_mul(f2_pack(__uint_as_float(w[2 * z]), __uint_as_float(w[2 * z + 1])), il2);
                w[z] = pack_bf16x2(f2_lo(y), f2_hi(y));
            }
            // Stores paced ~32 ns apart: issued back to back, the four epilogue warps' 32 KB backs up
            // the SM's memory pipeline and delays the MMA completion signals queued behind it (S(t)
            // was seen by the softmax ~5000 clk after its last MMA, ~300 clk with the pacing)
            if (store) {
#pragma unroll
                for (int u = 0; u < DH / 16; ++u) {
                    st_global_v8(d8 + (int64_t)u * a.H_q * 8, w + 8 * u);
                    if (u + 1 < DH / 16) __nanosleep(32);
                }
            }
            if (store) a.lse_part[(prow * a.k + slot) * a.H_q + h] = lse_row;
            if (row == 0) TL(7, qt);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
#undef TL
}

template <int DH, int G, bool F8>
cudaError_t launch_cfg(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t s, int n_sm)
{
    using C = AttnCfg<DH, G, F8>;
    const int smem = C::SMEM + (int)sizeof(AttnShared);
    static_assert(C::SMEM + sizeof(AttnShared) <= 227 * 1024, "shared memory budget");
    cudaError_t e =
        cudaFuncSetAttribute(sparse_attn_kernel<DH, G, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    sparse_attn_kernel<DH, G, F8><<<n_sm, 512, smem, s>>>(a, qmap, kmap, vmap);
    note_launch(1);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_dh(const AttnArgs& a, int G, const CUtensorMap& qmap, const CUtensorMap& kmap,
                      const CUtensorMap& vmap, cudaStream_t s, int n_sm)
{
    switch (G) {
    case 1: return launch_cfg<DH, 1, false>(a, qmap, kmap, vmap, s, n_sm);
    case 2: return launch_cfg<DH, 2, false>(a, qmap, kmap, vmap, s, n_sm);
    case 4: return launch_cfg<DH, 4, false>(a, qmap, kmap, vmap, s, n_sm);
    case 8: return launch_cfg<DH, 8, false>(a, qmap, kmap, vmap, s, n_sm);
    case 16: return launch_cfg<DH, 16, false>(a, qmap, kmap, vmap, s, n_sm);
    case 32: return launch_cfg<DH, 32, false>(a, qmap, kmap, vmap, s, n_sm);
    case 64: return launch_cfg<DH, 64, false>(a, qmap, kmap, vmap, s, n_sm);
    case 128: return launch_cfg<DH, 128, false>(a, qmap, kmap, vmap, s, n_sm);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace

cudaError_t launch_sparse_attn_fp8(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                                   const CUtensorMap& vmap, cudaStream_t s)
{
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (a.d_h != 128) return cudaErrorInvalidValue;
    switch (a.H_q / a.H_kv) {
    case 1: return launch_cfg<128, 1, true>(a, qmap, kmap, vmap, s, n_sm);
    case 2: return launch_cfg<128, 2, true>(a, qmap, kmap, vmap, s, n_sm);
    case 4: return launch_cfg<128, 4, true>(a, qmap, kmap, vmap, s, n_sm);
    case 8: return launch_cfg<128, 8, true>(a, qmap, kmap, vmap, s, n_sm);
    case 16: return launch_cfg<128, 16, true>(a, qmap, kmap, vmap, s, n_sm);
    default: return cudaErrorInvalidValue;
    }
}

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
