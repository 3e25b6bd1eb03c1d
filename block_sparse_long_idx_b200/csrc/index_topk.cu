// index_topk.cu -- fused Index Branch: index score tiles on tcgen05 tensor cores, block max-pool and
// exp-free Top-k in the epilogue ("MiniMax Sparse Attention" explainer, Figure 1 and section 05-1).
//
// Work item = (group r, pair of query tiles tA = 2u, tB = 2u+1), 128 query rows per tile. Tile t's
// rows all share the local block t, so their fully visible non-local blocks are b = 0 .. t-1. For
// each block b the CTA stages k_idx[b*128 .. +128, r, :] once (TMA) and issues two M=128, N=128
// MMAs (one per query tile) into TMEM, so one k_idx tile feeds 256 query rows. The epilogue thread
// that owns TMEM lane i reads its row's 128 scores, max-pools them, and offers the pooled score to
// its register Top-k list. The pooled score matrix never leaves the SM.
//
// Roles (384 threads): warp 0 = TMA producer, warps 1 and 2 = MMA issuers of tiles tA and tB (warp 1
// also owns TMEM), warps 4-7 = epilogue of tile tA, warps 8-11 = epilogue of tile tB. A thread
// stays busy about as long as the tensor pipe takes to run the MMAs it issues, plus tens of cycles
// per barrier wait and commit, so each tile has its own issuer and the barriers the two share
// (k_idx stage free, accumulator full, query tiles free) take one arrival from each. Persistent
// CTAs walk items in decreasing work order with a boustrophedon assignment.
#include <cstdio>

#include "common.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace msa {

namespace {

template <int DK>
struct IdxCfg {
    static constexpr int SWB = (DK * 2 >= 128) ? 128 : 64;    // swizzle row bytes
    static constexpr int CHUNK_COLS = SWB / 2;                  // elements per swizzle row
    static constexpr int NKC = (DK + CHUNK_COLS - 1) / CHUNK_COLS;
    static constexpr int CHUNK_BYTES = 128 * SWB;
    static constexpr int TILE_BYTES = CHUNK_BYTES * NKC;
    static constexpr int KSTEPS = DK / 16;
    static constexpr int NST = (200 * 1024 - 2 * TILE_BYTES) / TILE_BYTES > 8 ? 8
                                                                              : (200 * 1024 - 2 * TILE_BYTES) / TILE_BYTES;
    static constexpr int SMEM = 1024 + (2 + NST) * TILE_BYTES + 1024;
};

struct IdxShared {
    uint64_t q_full, q_empty, done;
    uint64_t kv_full[8], kv_empty[8];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

// Work item j: group r = j % H_kv and a pair u of query tiles of one sequence. The sequence's query
// rows are [row0, row0 + nrows) of the query tensors and start at block t0 of the sequence (t0 > 0
// when a prefix of the sequence is only in the key cache); its keys start at row krow0 of the key
// tensors. Tile A is the sequence's block tA = t0 + 2u (rows row0 + 256u ..), tile B is tA + 1; a
// row of tile t sees the blocks 0 .. t-1 in full. One sequence of N rows unless a.vitems.
struct IdxItem {
    int r, u, steps, tA;
    bool tbv;
    int row0, nrows, krow0;
};

__device__ __forceinline__ IdxItem item_at(const IndexTopkArgs& a, int j, int n_pairs)
{
    IdxItem it;
    it.r = j % a.H_kv;
    int t0 = 0;
    if (a.vitems) {
        const int2 v = a.vitems[j / a.H_kv];
        it.u = v.y;
        it.row0 = a.cu[v.x];
        it.nrows = a.cu[v.x + 1] - it.row0;
        it.krow0 = a.cu_k ? a.cu_k[v.x] : it.row0;
        if (a.cu_k) t0 = (a.cu_k[v.x + 1] - it.krow0 - it.nrows) / kBk; // cached prefix, whole blocks
    } else {
        it.u = n_pairs - 1 - j / a.H_kv;
        it.row0 = 0;
        it.nrows = (int)a.N;
        it.krow0 = 0;
    }
    const int n_qt = (it.nrows + kBk - 1) / kBk;
    it.tbv = (2 * it.u + 1) < n_qt;
    it.tA = t0 + 2 * it.u;
    it.steps = it.tbv ? it.tA + 1 : it.tA;
    return it;
}

__device__ __forceinline__ int item_for_round(int round, int cta, int P)
{
    return round * P + ((round & 1) ? (P - 1 - cta) : cta);
}

template <int DK>
__global__ void __launch_bounds__(384, 1)
    index_topk_kernel(IndexTopkArgs a, const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap)
{
    using C = IdxCfg<DK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sqA = smem;
    uint8_t* sqB = smem + C::TILE_BYTES;
    uint8_t* sk = smem + 2 * C::TILE_BYTES;
    IdxShared& sh = *reinterpret_cast<IdxShared*>(smem + (2 + C::NST) * C::TILE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qt = (int)((a.N + kBk - 1) / kBk);
    const int n_pairs = (n_qt + 1) / 2;
    const int n_items = (a.vitems ? a.n_vitems : n_pairs) * a.H_kv;
    const int P = gridDim.x, cta = blockIdx.x;
    volatile int* abort_flag = &sh.abort_flag;

    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_empty, 2);
        mbar_init(&sh.done, 2);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&sh.kv_full[s], 1);
            mbar_init(&sh.kv_empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.acc_full[b], 2);
            mbar_init(&sh.acc_empty[b], 8);
        }
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
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int gstep = 0, item_cnt = 0;
            bool ok = true;
            for (int round = 0; ok; ++round) {
                const int j = item_for_round(round, cta, P);
                if (j >= n_items) break;
                const IdxItem itm = item_at(a, j, n_pairs);
                const int r = itm.r, u = itm.u, steps = itm.steps;
                const bool tbv = itm.tbv;
                if (!wait_or_abort(&sh.q_empty, (item_cnt & 1) ^ 1, abort_flag, a.err, 1, kWaitLimit)) break;
                mbar_arrive_expect_tx(&sh.q_full, C::TILE_BYTES * (tbv ? 2 : 1));
                for (int c = 0; c < C::NKC; ++c) {
                    tma_load_3d(sqA + c * C::CHUNK_BYTES, &qmap, &sh.q_full, c * C::CHUNK_COLS, r,
                                itm.row0 + 2 * u * kBk);
                    if (tbv)
                        tma_load_3d(sqB + c * C::CHUNK_BYTES, &qmap, &sh.q_full, c * C::CHUNK_COLS, r,
                                    itm.row0 + (2 * u + 1) * kBk);
                }
                for (int b = 0; b < steps; ++b, ++gstep) {
                    const int s = gstep % C::NST;
                    if (!wait_or_abort(&sh.kv_empty[s], ((gstep / C::NST) & 1) ^ 1, abort_flag, a.err, 2, kWaitLimit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.kv_full[s], C::TILE_BYTES);
                    for (int c = 0; c < C::NKC; ++c)
                        tma_load_3d(sk + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &kmap, &sh.kv_full[s],
                                    c * C::CHUNK_COLS, r, itm.krow0 + b * kBk);
                }
                ++item_cnt;
            }
            // drain: every issued k_idx load has landed before the CTA may exit
            for (int g = gstep - 1; g >= 0 && g >= gstep - C::NST; --g)
                drain_wait(&sh.kv_full[g % C::NST], (g / C::NST) & 1, a.err, 7, kWaitLimit);
            if (item_cnt > 0) drain_wait(&sh.q_full, (item_cnt - 1) & 1, a.err, 8, kWaitLimit);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------------------------ MMA issuers (warp 1: tile A, 2: tile B)
        const int tsel = warp - 1;
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
            const uint32_t aA = smem_u32(sqA), aB = smem_u32(sqB), ak = smem_u32(sk);
            int gstep = 0, acc_cnt = 0, item_cnt = 0;
            bool ok = true;
            for (int round = 0; ok; ++round) {
                const int j = item_for_round(round, cta, P);
                if (j >= n_items) break;
                const IdxItem itm = item_at(a, j, n_pairs);
                const int steps = itm.steps;
                const bool tbv = itm.tbv;
                if (!poll_or_abort(&sh.q_full, item_cnt & 1, abort_flag, a.err, 3, kWaitLimit)) break;
                tc_fence_after();
                for (int b = 0; b < steps; ++b, ++gstep, ++acc_cnt) {
                    const int s = gstep % C::NST;
                    const int buf = acc_cnt & 1;
                    if (!poll_or_abort(&sh.kv_full[s], (gstep / C::NST) & 1, abort_flag, a.err, 4, kWaitLimit) ||
                        !poll_or_abort(&sh.acc_empty[buf], ((acc_cnt >> 1) & 1) ^ 1, abort_flag, a.err, 5, kWaitLimit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t kb = ak + s * C::TILE_BYTES;
                    // tile A sees blocks 0 .. tA-1, tile B (when present) blocks 0 .. tA
                    const bool mine = tsel == 0 ? b < itm.tA : tbv;
                    if (mine) {
#pragma unroll
                        for (int ks = 0; ks < C::KSTEPS; ++ks) {
                            const int col = ks * 16;
                            const uint32_t off = (col / C::CHUNK_COLS) * C::CHUNK_BYTES + (col % C::CHUNK_COLS) * 2;
                            const uint64_t kd = desc_kmajor(kb + off, C::SWB);
                            mma_ss(tmem + tsel * 256 + buf * 128, desc_kmajor((tsel ? aB : aA) + off, C::SWB), kd,
                                   idesc, ks > 0);
                        }
                    }
                    tc_commit(&sh.kv_empty[s]);
                    tc_commit(&sh.acc_full[buf]);
                }
                tc_commit(&sh.q_empty);
                ++item_cnt;
            }
            tc_commit(&sh.done);
            drain_wait(&sh.done, 0, a.err, 9, kWaitLimit);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue: pool + Top-k
        const int e = (warp - 4) >> 2;   // 0: tile tA, 1: tile tB
        const int quarter = warp & 3;    // TMEM lane quarter
        const int row = quarter * 32 + lane;
        int acc_cnt = 0;
        for (int round = 0;; ++round) {
            const int j = item_for_round(round, cta, P);
            if (j >= n_items) break;
            const IdxItem itm = item_at(a, j, n_pairs);
            const int r = itm.r, u = itm.u, steps = itm.steps;
            const bool tbv = itm.tbv;
            const int tile = itm.tA + e; // the sequence's block of this tile's rows
            const bool active = (e == 0) || tbv;
            TopkList list;
            list.init(a.k - 1);
            bool ok = true;
            for (int b = 0; b < steps; ++b, ++acc_cnt) {
                const int buf = acc_cnt & 1;
                if (!wait_or_abort(&sh.acc_full[buf], (acc_cnt >> 1) & 1, abort_flag, a.err, 6, kWaitLimit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (active && (e == 1 || b < itm.tA)) {
                    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (e ? 256 : 0) + buf * 128;
                    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, m2 = -CUDART_INF_F, m3 = -CUDART_INF_F;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t x[32], y[32];
                        tmem_ld32(taddr + half * 64, x);
                        tmem_ld32(taddr + half * 64 + 32, y);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            m0 = max3f(m0, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
                            m1 = max3f(m1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
                            m2 = max3f(m2, __uint_as_float(y[c]), __uint_as_float(y[c + 1]));
                            m3 = max3f(m3, __uint_as_float(y[c + 2]), __uint_as_float(y[c + 3]));
                        }
                    }
                    list.offer_ascending(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), b); // blocks arrive in ascending order
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.acc_empty[buf]);
            }
            if (!ok) break;
            if (active) {
                const int il = (2 * u + e) * kBk + row; // row among the sequence's query rows
                if (il < itm.nrows)
                    emit_selection(list, tile, a.k, a.block_idx + ((int64_t)r * a.N + itm.row0 + il) * a.k);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DK>
cudaError_t launch_dk(const IndexTopkArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap, cudaStream_t s)
{
    using C = IdxCfg<DK>;
    static_assert(C::SMEM + sizeof(IdxShared) <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(index_topk_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM + (int)sizeof(IdxShared));
    if (e != cudaSuccess) return e;
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int n_qt = (int)((a.N + kBk - 1) / kBk);
    const int n_items = (a.vitems ? a.n_vitems : (n_qt + 1) / 2) * a.H_kv;
    const int grid = n_items < n_sm ? n_items : n_sm;
    index_topk_kernel<DK><<<grid, 384, C::SMEM + sizeof(IdxShared), s>>>(a, qmap, kmap);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_index_topk(const IndexTopkArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              cudaStream_t s)
{
    switch (a.d_idx) {
    case 32: return launch_dk<32>(a, qmap, kmap, s);
    case 64: return launch_dk<64>(a, qmap, kmap, s);
    case 128: return launch_dk<128>(a, qmap, kmap, s);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace msa
