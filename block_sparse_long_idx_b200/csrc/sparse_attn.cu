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
//                                     TMEM as bf16 over the S columns
//   O = P V                           tcgen05.mma, A = P (TMEM), B = V (smem, MN-major)
//   partial[p, slot, h] = O / rowsum, lse = rowmax*scale + log(rowsum)
// A work item covers one KV block only, so no running-max rescaling is needed. Stage 2
// (combine.cu) merges the <= k partials of every (row, head) through their lse.
//
// Roles (384 threads): warp 0 = K/V TMA producer, warp 1 = MMA issuer + TMEM owner, warp 2 = Q
// gather (one TMA box per position, issued by the 32 lanes in parallel), warps 4-7 and 8-11 =
// softmax + epilogue for even and odd tiles. TMEM: S/P of tile buffer i at columns [128 i, +128),
// O of buffer i at [256 + 128 i, +d_h). Barriers per buffer: s_full (S written), p_full (P
// written), o_full (O written, which also frees S/P), o_free (epilogue has read O).
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
    static constexpr int NQ = 3;                 // Q stages
    static constexpr int SMEM = 1024 + NQ * TILE + 4 * TILE;
};

struct AttnShared {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[3], q_empty[3];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr uint32_t kNegInfBits = 0xff800000u;
constexpr int REG_LO = 56, REG_HI = 216; // 128 * 56 + 256 * 216 = 62464 <= 384 * 168

template <int DH, int G>
__global__ void __launch_bounds__(384, 1)
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
    const int P = gridDim.x, cta = blockIdx.x;
    const int64_t Nk = a.N * a.k;
    volatile int* abort_flag = &sh.abort_flag;
    const int j_begin = a.window_items[a.w0] + cta;
    const int j_end = a.window_items[a.w1];
    const bool tl_on = a.timeline != nullptr && cta == 0;
#define TL(slot, tile)                                                                                    \
    do {                                                                                                  \
        if (tl_on && (tile) < a.timeline_tiles) a.timeline[(int64_t)(tile) * 10 + (slot)] = clock64();    \
    } while (0)

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.kv_full[i], 1);
            mbar_init(&sh.kv_empty[i], 1);
            mbar_init(&sh.s_full[i], 1);
            mbar_init(&sh.p_full[i], 4);
            mbar_init(&sh.o_full[i], 1);
            mbar_init(&sh.o_free[i], 4);
        }
        for (int i = 0; i < NQ; ++i) {
            mbar_init(&sh.q_full[i], 1);
            mbar_init(&sh.q_empty[i], 1);
        }
        mbar_init(&sh.done, 1);
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

    // Register split (each warpgroup executes its own setmaxnreg inside its branch): 384 threads x
    // 168 launch registers = 64512 >= producer warpgroup 128 x REG_LO + softmax warpgroups 256 x REG_HI.
    if (warp < 4) {
        reg_dealloc<REG_LO>();
    if (warp == 0) {
        // ------------------------------------------------------------ K/V producer
        if (lane == 0) {
            int it = 0;
            for (int j = j_begin; j < j_end; j += P, ++it) {
                const msa_work_item item = a.items[j];
                const int s = it & 1;
                if (!wait_or_abort(&sh.kv_empty[s], ((it >> 1) & 1) ^ 1, abort_flag, a.err, 20, kWaitLimit)) break;
                mbar_arrive_expect_tx(&sh.kv_full[s], 2 * C::TILE);
                for (int c = 0; c < C::NKC; ++c) {
                    tma_load_3d(sK + s * C::TILE + c * C::CHUNK, &kmap, &sh.kv_full[s], c * 64, item.r, item.b * kBk);
                    tma_load_3d(sV + s * C::TILE + c * C::CHUNK, &vmap, &sh.kv_full[s], c * 64, item.r, item.b * kBk);
                }
            }
            for (int g = it - 1; g >= 0 && g >= it - 2; --g) mbar_wait(&sh.kv_full[g & 1], (g >> 1) & 1, kWaitLimit);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ Q gather (TMA per position)
        int qt = 0;
        bool ok = true;
        for (int j = j_begin; j < j_end && ok; j += P) {
            const msa_work_item item = a.items[j];
            const int32_t* ent = a.entries + (int64_t)item.r * Nk + item.start;
            const int ntiles = (item.len + PPT - 1) / PPT;
            for (int t = 0; t < ntiles; ++t, ++qt) {
                const int qs = qt % NQ;
                const int npos = min(PPT, item.len - t * PPT);
                // fetch this tile's rows before waiting for the stage
                int prow[(PPT + 31) / 32];
#pragma unroll
                for (int u = 0; u < (PPT + 31) / 32; ++u) {
                    const int pl = lane + 32 * u;
                    prow[u] = pl < npos ? ent[t * PPT + pl] / a.k : 0;
                }
                int w_ok = 1;
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
                            tma_load_3d(sQ + qs * C::TILE + c * C::CHUNK + pl * G * 128, &qmap, &sh.q_full[qs], c * 64,
                                        item.r * G, prow[u]);
                    }
                }
                if (lane == 0) TL(1, qt);
            }
        }
        if (lane == 0)
            for (int g = qt - 1; g >= 0 && g >= qt - NQ; --g) mbar_wait(&sh.q_full[g % NQ], (g / NQ) & 1, kWaitLimit);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idPV = idesc_bf16_f32(128, DH, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            int qt = 0, it = 0;
            int prev_qt = -1, prev_kvs = 0;
            bool prev_last = false, ok = true;
            // O(pqt) = P(pqt) V: needs P written and the O buffer read by the epilogue of pqt-2
            auto issue_pv = [&](int pqt, int pkvs, bool plast) -> bool {
                const int pb = pqt & 1;
                if (!wait_or_abort(&sh.p_full[pb], (pqt >> 1) & 1, abort_flag, a.err, 22, kWaitLimit)) return false;
                if (!wait_or_abort(&sh.o_free[pb], ((pqt >> 1) & 1) ^ 1, abort_flag, a.err, 28, kWaitLimit))
                    return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem + 256 + pb * 128, tmem + pb * 128 + ks * 8,
                           smem_desc(aV + pkvs * C::TILE + ks * 2048, C::CHUNK, 1024, 128), idPV, ks > 0);
                tc_commit(&sh.o_full[pb]);
                if (plast) tc_commit(&sh.kv_empty[pkvs]);
                TL(3, pqt);
                return true;
            };
            for (int j = j_begin; j < j_end && ok; j += P, ++it) {
                const msa_work_item item = a.items[j];
                const int kvs = it & 1;
                const int ntiles = (item.len + PPT - 1) / PPT;
                if (!wait_or_abort(&sh.kv_full[kvs], (it >> 1) & 1, abort_flag, a.err, 23, kWaitLimit)) break;
                TL(8, qt);
                for (int t = 0; t < ntiles; ++t, ++qt) {
                    const int buf = qt & 1, qs = qt % NQ;
                    // S/P buffer is free once PV(qt-2) has completed
                    if (!wait_or_abort(&sh.q_full[qs], (qt / NQ) & 1, abort_flag, a.err, 24, kWaitLimit) ||
                        (qt >= 2 && !wait_or_abort(&sh.o_full[buf], ((qt >> 1) & 1) ^ 1, abort_flag, a.err, 25,
                                                   kWaitLimit))) {
                        ok = false;
                        break;
                    }
                    TL(9, qt);
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < DH / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
                        mma_ss(tmem + buf * 128, desc_kmajor(aQ + qs * C::TILE + off, 128),
                               desc_kmajor(aK + kvs * C::TILE + off, 128), idS, ks > 0);
                    }
                    tc_commit(&sh.s_full[buf]);
                    tc_commit(&sh.q_empty[qs]);
                    TL(2, qt);
                    if (prev_qt >= 0 && !issue_pv(prev_qt, prev_kvs, prev_last)) {
                        ok = false;
                        break;
                    }
                    prev_qt = qt;
                    prev_kvs = kvs;
                    prev_last = (t == ntiles - 1);
                }
            }
            if (ok && prev_qt >= 0) issue_pv(prev_qt, prev_kvs, prev_last);
            tc_commit(&sh.done);
            mbar_wait(&sh.done, 0, kWaitLimit);
        }
    }
    } else {
        reg_alloc<REG_HI>();
        // ------------------------------------------------------------ softmax + epilogue
        const int beta = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int pl = row / G, hh = row % G;
        const float scale = rsqrtf((float)DH);
        const float sl2 = scale * 1.4426950408889634f;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        int qt = 0;
        bool ok = true;
        for (int j = j_begin; j < j_end && ok; j += P) {
            const msa_work_item item = a.items[j];
            const int32_t* ent = a.entries + (int64_t)item.r * Nk + item.start;
            const int ntiles = (item.len + PPT - 1) / PPT;
            for (int t = 0; t < ntiles; ++t, ++qt) {
                if ((qt & 1) != beta) continue;
                const int buf = beta;
                const int idx = t * PPT + pl;
                const bool valid = idx < item.len;
                const int32_t e = valid ? ent[idx] : 0;
                const int p = e / a.k;
                const int slot = e - p * a.k;
                const int limit = valid ? min(127, p - item.b * kBk) : 127;
                if (!wait_or_abort(&sh.s_full[buf], (qt >> 1) & 1, abort_flag, a.err, 26, kWaitLimit)) {
                    ok = false;
                    break;
                }
                if (row == 0) TL(4, qt);
                tc_fence_after();
                const uint32_t sadr = lane_base + buf * 128;
                uint32_t s[128];
                tmem_ld32_at<0>(sadr, s);
                tmem_ld32_at<32>(sadr + 32, s);
                tmem_ld32_at<64>(sadr + 64, s);
                tmem_ld32_at<96>(sadr + 96, s);
                tmem_ld_wait();
                if (limit < 127) { // the query's own block: keys after the query are invisible
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > limit) s[c] = kNegInfBits;
                }
                // row max: 3-input max tree
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
                tmem_st_wait();
                const float l = f2_lo(l2) + f2_hi(l2);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.p_full[buf]);
                if (row == 0) TL(5, qt);

                // epilogue: O / l -> partial slot, lse
                if (!wait_or_abort(&sh.o_full[buf], (qt >> 1) & 1, abort_flag, a.err, 27, kWaitLimit)) {
                    ok = false;
                    break;
                }
                if (row == 0) TL(6, qt);
                tc_fence_after();
                const uint32_t oadr = lane_base + 256 + buf * 128;
                uint32_t o[DH];
                tmem_ld32_at<0>(oadr, o);
                tmem_ld32_at<32>(oadr + 32, o);
                if constexpr (DH == 128) {
                    tmem_ld32_at<64 % DH>(oadr + 64, o);
                    tmem_ld32_at<96 % DH>(oadr + 96, o);
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.o_free[buf]);
                const float inv_l = 1.f / l;
                const int h = item.r * G + hh;
                const int64_t prow = (int64_t)(p - a.row0);
                bool store = valid;
                if (valid && (prow < 0 || prow >= a.rows_pass || slot < 0 || slot >= a.k)) {
                    report_error(a.err, MSA_ERR_DEVICE_CHECK, 300); // entry outside this pass: skip it
                    store = false;
                }
                if (store) {
                    // partial layout [row][slot][d_h/8][H_q][8]: the G heads of a position are adjacent
                    // 16-byte units, so each warp-wide store writes contiguous runs
                    uint4* d4 = reinterpret_cast<uint4*>(a.o_part + (prow * a.k + slot) * (int64_t)a.H_q * DH) + h;
                    const uint64_t il2 = f2_pack(inv_l, inv_l);
#pragma unroll
                    for (int q = 0; q < DH / 8; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            const uint64_t y = f2_mul(f2_pack(__uint_as_float(o[8 * q + 2 * z]),
                                                              __uint_as_float(o[8 * q + 2 * z + 1])),
                                                      il2);
                            w[z] = pack_bf16x2(f2_lo(y), f2_hi(y));
                        }
                        d4[q * a.H_q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    a.lse_part[(prow * a.k + slot) * a.H_q + h] = m * scale + logf(l);
                }
                if (row == 0) TL(7, qt);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}
#undef TL

template <int DH, int G>
cudaError_t launch_cfg(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t s, int n_sm)
{
    using C = AttnCfg<DH>;
    const int smem = C::SMEM + (int)sizeof(AttnShared);
    static_assert(AttnCfg<DH>::SMEM + sizeof(AttnShared) <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<DH, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    sparse_attn_kernel<DH, G><<<n_sm, 384, smem, s>>>(a, qmap, kmap, vmap);
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
