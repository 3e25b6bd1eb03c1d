// sparse_attn.cu -- KV-outer block-sparse attention, stage 1 of the two-stage forward
// ("MiniMax Sparse Attention" explainer, section 05-2).
//
// Each work item is one (group r, KV block b, chunk of the rows that selected b). Its K and V blocks
// are staged in shared memory once by TMA; the rows are processed in 128-row tensor-core tiles made
// of 128/G query positions x G heads ("query concatenation"), each position's G heads gathered by
// one TMA box from q[p, r*G .. r*G+G, :]. Per tile:
//   S = Q K^T                         tcgen05.mma, A = Q (smem), B = K (smem), D in TMEM
//   P = exp(S*scale - rowmax)         softmax warps, thread = TMEM lane = tile row, causal mask on
//                                     the query's own block, P written back to TMEM as bf16
//   O = P V                           tcgen05.mma, A = P (TMEM), B = V (smem, MN-major)
//   partial[p, slot, h] = O / rowsum, lse = rowmax*scale + log(rowsum)
// A work item covers one KV block only, so no running-max rescaling is needed. Stage 2
// (combine.cu) merges the <= k partials of every (row, head) through their lse.
//
// Roles (384 threads): warp 0 = K/V TMA producer, warp 1 = MMA issuer + TMEM owner, warp 2 = Q
// gather (one TMA box per position, issued by the 32 lanes in parallel), warps 4-7 and 8-11 =
// softmax + epilogue for even and odd tiles (TMEM ping-pong: S/P at cols [256*buf, +128), O at
// [256*buf + 128, +d_h)), so one tile's softmax overlaps the other tile's MMAs.
#include "common.cuh"
#include <math_constants.h>

#include "sm100.cuh"

namespace msa {

namespace {

template <int DH>
struct AttnCfg {
    static constexpr int NKC = DH / 64;          // 64-column (128-byte) chunks
    static constexpr int CHUNK = 128 * 128;      // bytes per chunk of a 128-row tile
    static constexpr int TILE = NKC * CHUNK;     // Q, K or V tile bytes
    static constexpr int NQ = 2;                 // Q stages
    static constexpr int SMEM = 1024 + NQ * TILE + 4 * TILE + 1024;
};

struct AttnShared {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], p_full[2], o_full[2], tm_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int DH, int G>
__global__ void __launch_bounds__(384, 1)
    sparse_attn_kernel(AttnArgs a, const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap)
{
    using C = AttnCfg<DH>;
    constexpr int PPT = 128 / G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                       // [NQ][TILE]
    uint8_t* sK = smem + C::NQ * C::TILE;     // [2][TILE]
    uint8_t* sV = sK + 2 * C::TILE;           // [2][TILE]
    AttnShared& sh = *reinterpret_cast<AttnShared*>(sV + 2 * C::TILE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, cta = blockIdx.x;
    const int64_t Nk = a.N * a.k;
    volatile int* abort_flag = &sh.abort_flag;
    const int j_begin = a.window_items[a.w0] + cta;
    const int j_end = a.window_items[a.w1];

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.kv_full[i], 1);
            mbar_init(&sh.kv_empty[i], 1);
            mbar_init(&sh.q_full[i], 1);
            mbar_init(&sh.q_empty[i], 1);
            mbar_init(&sh.s_full[i], 1);
            mbar_init(&sh.p_full[i], 4);
            mbar_init(&sh.o_full[i], 1);
            mbar_init(&sh.tm_empty[i], 4);
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
                const int qs = qt & 1;
                int w_ok = 1;
                if (lane == 0)
                    w_ok = wait_or_abort(&sh.q_empty[qs], ((qt >> 1) & 1) ^ 1, abort_flag, a.err, 21, kWaitLimit);
                w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                const int npos = min(PPT, item.len - t * PPT);
                if (lane == 0) mbar_arrive_expect_tx(&sh.q_full[qs], npos * G * DH * 2);
                __syncwarp();
                for (int pl = lane; pl < npos; pl += 32) {
                    const int32_t e = ent[t * PPT + pl];
                    const int p = e / a.k;
#pragma unroll
                    for (int c = 0; c < C::NKC; ++c)
                        tma_load_3d(sQ + qs * C::TILE + c * C::CHUNK + pl * G * 128, &qmap, &sh.q_full[qs], c * 64,
                                    item.r * G, p);
                }
            }
        }
        if (lane == 0)
            for (int g = qt - 1; g >= 0 && g >= qt - 2; --g) mbar_wait(&sh.q_full[g & 1], (g >> 1) & 1, kWaitLimit);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idPV = idesc_bf16_f32(128, DH, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            int qt = 0, it = 0;
            int prev_qt = -1, prev_kvs = 0;
            bool prev_last = false, ok = true;
            auto issue_pv = [&](int pqt, int pkvs, bool plast) -> bool {
                const int pb = pqt & 1;
                if (!wait_or_abort(&sh.p_full[pb], (pqt >> 1) & 1, abort_flag, a.err, 22, kWaitLimit)) return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem + pb * 256 + 128, tmem + pb * 256 + ks * 8,
                           smem_desc(aV + pkvs * C::TILE + ks * 2048, C::CHUNK, 1024, 128), idPV, ks > 0);
                tc_commit(&sh.o_full[pb]);
                if (plast) tc_commit(&sh.kv_empty[pkvs]);
                return true;
            };
            for (int j = j_begin; j < j_end && ok; j += P, ++it) {
                const msa_work_item item = a.items[j];
                const int kvs = it & 1;
                const int ntiles = (item.len + PPT - 1) / PPT;
                if (!wait_or_abort(&sh.kv_full[kvs], (it >> 1) & 1, abort_flag, a.err, 23, kWaitLimit)) break;
                for (int t = 0; t < ntiles; ++t, ++qt) {
                    const int buf = qt & 1, qs = qt & 1;
                    if (!wait_or_abort(&sh.q_full[qs], (qt >> 1) & 1, abort_flag, a.err, 24, kWaitLimit) ||
                        !wait_or_abort(&sh.tm_empty[buf], ((qt >> 1) & 1) ^ 1, abort_flag, a.err, 25, kWaitLimit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < DH / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
                        mma_ss(tmem + buf * 256, desc_kmajor(aQ + qs * C::TILE + off, 128),
                               desc_kmajor(aK + kvs * C::TILE + off, 128), idS, ks > 0);
                    }
                    tc_commit(&sh.s_full[buf]);
                    tc_commit(&sh.q_empty[qs]);
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
    } else if (warp >= 4) {
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
                tc_fence_after();
                const uint32_t sadr = lane_base + buf * 256;
                // pass 1: row max over the visible keys
                float m = -CUDART_INF_F;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t x[32], y[32];
                    tmem_ld32(sadr + h2 * 64, x);
                    tmem_ld32(sadr + h2 * 64 + 32, y);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (h2 * 64 + c <= limit) m = fmaxf(m, __uint_as_float(x[c]));
                        if (h2 * 64 + 32 + c <= limit) m = fmaxf(m, __uint_as_float(y[c]));
                    }
                }
                // pass 2: exponentials, row sum, P (bf16) into TMEM over the consumed S columns
                const float ms = m * sl2;
                float l = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t x[32], pk[16];
                    tmem_ld32(sadr + c4 * 32, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int k0 = c4 * 32 + 2 * q;
                        const float e0 = k0 <= limit ? ex2_approx(fmaf(__uint_as_float(x[2 * q]), sl2, -ms)) : 0.f;
                        const float e1 =
                            k0 + 1 <= limit ? ex2_approx(fmaf(__uint_as_float(x[2 * q + 1]), sl2, -ms)) : 0.f;
                        l += e0 + e1;
                        pk[q] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(sadr + c4 * 16, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.p_full[buf]);

                // epilogue: O / l -> partial slot, lse
                if (!wait_or_abort(&sh.o_full[buf], (qt >> 1) & 1, abort_flag, a.err, 27, kWaitLimit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float inv_l = 1.f / l;
                const int h = item.r * G + hh;
                const int64_t prow = (int64_t)(p - a.row0);
                bool store = valid;
                if (valid && (prow < 0 || prow >= a.rows_pass || slot < 0 || slot >= a.k)) {
                    report_error(a.err, MSA_ERR_DEVICE_CHECK, 300); // entry outside this pass: skip it
                    store = false;
                }
                uint16_t* dst = a.o_part + ((prow * a.k + slot) * a.H_q + h) * (int64_t)DH;
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(sadr + 128 + c * 32, x);
                    tmem_ld_wait();
                    uint4 v[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        v[q].x = pack_bf16x2(__uint_as_float(x[8 * q + 0]) * inv_l, __uint_as_float(x[8 * q + 1]) * inv_l);
                        v[q].y = pack_bf16x2(__uint_as_float(x[8 * q + 2]) * inv_l, __uint_as_float(x[8 * q + 3]) * inv_l);
                        v[q].z = pack_bf16x2(__uint_as_float(x[8 * q + 4]) * inv_l, __uint_as_float(x[8 * q + 5]) * inv_l);
                        v[q].w = pack_bf16x2(__uint_as_float(x[8 * q + 6]) * inv_l, __uint_as_float(x[8 * q + 7]) * inv_l);
                    }
                    if (store) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                        for (int q = 0; q < 4; ++q) d4[q] = v[q];
                    }
                }
                if (store) a.lse_part[(prow * a.k + slot) * a.H_q + h] = m * scale + logf(l);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.tm_empty[buf]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DH, int G>
cudaError_t launch_cfg(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t s, int n_sm)
{
    using C = AttnCfg<DH>;
    const int smem = C::SMEM + (int)sizeof(AttnShared);
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
