// decode.cu -- MSA decode: one query token per sequence against a KV cache ("MiniMax Sparse
// Attention" abstract: prefill and decoding speedups; explainer Figure 4 right).
//
// Sequence beta's query sits at position i = len - 1; its selection and attention are those of
// prefill row i (explainer Figure 1 and section 05). Three kernels, then the shared combine:
//   1. decode_pool   : index scores q_idx . k_idx over the whole k_idx cache, block max-pooled.
//                      HBM-bound streaming (~len*H_kv*d_idx*2 bytes per sequence): whole cache blocks
//                      by bulk copy into a 3-stage shared-memory ring per SM, scored on CUDA cores (a
//                      warp-wide load covers whole cache rows, each lane dots 8 elements, lanes of a
//                      group reduce with shuffles). Exact for integer-valued index inputs.
//   2. decode_topk   : per (sequence, group) one warp; each lane keeps a register Top-(k-1) list over
//                      its 1/32 of the pooled row, then a warp-shuffle merge (explainer section 05-1)
//                      and the forced local block.
//   3. decode_attn   : per (sequence, group, slot) one CTA: the G query heads (padded to 16 rows)
//                      against the slot's 128-key block with mma.sync m16n8k16 (a 16-row problem is
//                      below the 64/128-row tcgen05 tile and the kernel is bound by reading K/V),
//                      writing a partial (normalised output, lse) like prefill's stage 1.
#include <math_constants.h>

#include "common.cuh"
#include "mma_sync.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace msa {

namespace {

constexpr int kPoolConsumers = 8;                  // scoring warps of a pooling CTA
constexpr int kPoolStages = 3;                     // k_idx cache blocks in flight per SM
constexpr int kPoolStageBytes = kBk * 512;         // one block of rows up to 512 bytes (H_kv * d_idx <= 256)

struct PoolShared {
    uint64_t full[kPoolStages], empty[kPoolStages];
    float pmax[kPoolStages][kPoolConsumers][32]; // [stage][warp][group]: the warp's rows' maximum
    int abort_flag;
};
constexpr int kPoolSmem = kPoolStages * kPoolStageBytes + (int)sizeof(PoolShared);

__device__ __forceinline__ int seq_local_block(int len) { return (len - 1) / kBk; }

// ----------------------------------------------------------------------------------- 1. pooling
// Work balance: sequences have very different lengths, so the fully visible blocks of all
// sequences form one flattened list (prefix[beta] = blocks of the sequences before beta) and every
// warp of a persistent grid streams an equal contiguous slice of it.
__global__ void __launch_bounds__(1024) decode_prefix_kernel(DecodeArgs a)
{
    __shared__ int64_t warp_sum[32];
    __shared__ int64_t carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        carry = 0;
        a.blk_prefix[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < a.B; base += 1024) {
        const int beta = base + tid;
        int64_t n = 0;
        if (beta < a.B) {
            const int len = a.lens[beta];
            n = (len >= 1 && len <= a.L_max) ? seq_local_block(len) : 0;
        }
        int64_t x = n; // inclusive scan: warp, then across warps
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int64_t w = warp_sum[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sum[lane] = w;
        }
        __syncthreads();
        const int64_t incl = carry + x + (warp > 0 ? warp_sum[warp - 1] : 0);
        if (beta < a.B) a.blk_prefix[beta + 1] = incl;
        __syncthreads();
        if (tid == 1023) carry = incl;
        __syncthreads();
    }
}

// One CTA per SM streams an equal contiguous slice of the flattened block list. Its producer thread
// keeps kPoolStages whole blocks of the k_idx cache in flight (one bulk copy each: a block's 128 rows
// are contiguous), and kPoolConsumers warps score 128 / kPoolConsumers rows of every block from
// shared memory: a warp-wide 16-byte load per lane covers whole cache rows, each lane dots its 8
// elements, the lanes of a group reduce by shuffles. Each warp leaves its per-group maxima in shared
// memory; the producer reduces them and writes the pooled scores before it refills the stage.
__global__ void __launch_bounds__((kPoolConsumers + 1) * 32, 1) decode_pool_kernel(DecodeArgs a, int nb_max)
{
    extern __shared__ __align__(1024) uint8_t pool_smem[];
    PoolShared& sh = *reinterpret_cast<PoolShared*>(pool_smem + kPoolStages * kPoolStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row_elems = (int64_t)a.H_kv * a.d_idx;
    const uint32_t blk_bytes = (uint32_t)(kBk * row_elems * 2);
    const int64_t total = a.blk_prefix[a.B];
    const int64_t g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPoolStages; ++i) {
            mbar_init(&sh.full[i], 1);
            mbar_init(&sh.empty[i], kPoolConsumers);
        }
        sh.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (g0 >= g1) return;
    volatile int* abort_flag = &sh.abort_flag;
    // the sequence holding block g0: the last beta with prefix[beta] <= g0
    int lo = 0, hi = a.B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.blk_prefix[mid] <= g0) lo = mid; else hi = mid - 1;
    }
    if (warp == kPoolConsumers) {
        // ---------------------------------------------------------------- producer (lane 0)
        if (lane != 0) return;
        int pend_beta[kPoolStages], pend_b[kPoolStages];
        auto flush = [&](int s) { // all consumers are done with stage s: its block's pooled scores
            for (int r = 0; r < a.H_kv; ++r) {
                float m = sh.pmax[s][0][r];
#pragma unroll
                for (int w = 1; w < kPoolConsumers; ++w) m = fmaxf(m, sh.pmax[s][w][r]);
                a.pooled[((int64_t)pend_beta[s] * a.H_kv + r) * nb_max + pend_b[s]] = m;
            }
        };
        int beta = lo;
        bool ok = true;
        int64_t n = 0;
        for (int64_t g = g0; g < g1; ++g, ++n) {
            const int s = (int)(n % kPoolStages);
            if (n >= kPoolStages) {
                if (!wait_or_abort(&sh.empty[s], (uint32_t)((n / kPoolStages - 1) & 1), abort_flag, a.err, 50,
                                   kWaitLimit)) {
                    ok = false;
                    break;
                }
                flush(s);
            }
            while (a.blk_prefix[beta + 1] <= g) ++beta;
            const int b = (int)(g - a.blk_prefix[beta]);
            pend_beta[s] = beta;
            pend_b[s] = b;
            mbar_arrive_expect_tx(&sh.full[s], blk_bytes);
            bulk_load(pool_smem + s * kPoolStageBytes,
                      a.k_idx_cache + ((int64_t)beta * a.L_max + (int64_t)b * kBk) * row_elems, blk_bytes,
                      &sh.full[s]);
        }
        // the last stages: flush them, or (after an abort) wait for their copies before the CTA exits
        for (int64_t m = n > kPoolStages ? n - kPoolStages : 0; m < n; ++m) {
            const int s = (int)(m % kPoolStages);
            if (ok && wait_or_abort(&sh.empty[s], (uint32_t)((m / kPoolStages) & 1), abort_flag, a.err, 51,
                                    kWaitLimit))
                flush(s);
            else
                drain_wait(&sh.full[s], (uint32_t)((m / kPoolStages) & 1), a.err, 52, kWaitLimit);
        }
        return;
    }
    // -------------------------------------------------------------------- consumers
    const int lanes_per_pos = (int)(row_elems / 8);
    const int pos_per_step = 32 / lanes_per_pos;
    const int lanes_per_group = a.d_idx / 8;
    const int sub = lane % lanes_per_pos;
    const int r = sub / lanes_per_group;
    const int pos_lane = lane / lanes_per_pos;
    constexpr int kRows = kBk / kPoolConsumers; // rows of every block this warp scores
    int beta = lo - 1;
    float qf[8];
    int64_t n = 0;
    for (int64_t g = g0; g < g1; ++g, ++n) {
        const int s = (int)(n % kPoolStages);
        if (beta < lo || a.blk_prefix[beta + 1] <= g) { // entering the next sequence that owns blocks
            beta = beta < lo ? lo : beta + 1;
            while (a.blk_prefix[beta + 1] <= g) ++beta;
            const uint4 qv = *reinterpret_cast<const uint4*>(a.q_idx + ((int64_t)beta * a.H_kv) * a.d_idx + sub * 8);
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                qf[2 * q] = __uint_as_float(qw[q] << 16);
                qf[2 * q + 1] = __uint_as_float(qw[q] & 0xFFFF0000u);
            }
        }
        if (!wait_or_abort(&sh.full[s], (uint32_t)((n / kPoolStages) & 1), abort_flag, a.err, 53, kWaitLimit)) break;
        const uint16_t* blk = reinterpret_cast<const uint16_t*>(pool_smem + s * kPoolStageBytes) + sub * 8;
        float m = -CUDART_INF_F;
        for (int j0 = 0; j0 < kRows; j0 += 8 * pos_per_step) {
            uint4 kv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * pos_per_step + pos_lane;
                kv[u] = j < kRows ? *reinterpret_cast<const uint4*>(blk + (int64_t)(warp * kRows + j) * row_elems)
                                  : make_uint4(0u, 0u, 0u, 0u);
            }
            float sc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t kw[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc = fmaf(qf[2 * q], __uint_as_float(kw[q] << 16), acc);
                    acc = fmaf(qf[2 * q + 1], __uint_as_float(kw[q] & 0xFFFF0000u), acc);
                }
                sc[u] = acc;
            }
            for (int o = lanes_per_group >> 1; o > 0; o >>= 1) {
#pragma unroll
                for (int u = 0; u < 8; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j0 + u * pos_per_step < kRows) m = fmaxf(m, sc[u]);
        }
        for (int o = lanes_per_pos; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane < lanes_per_pos && (sub % lanes_per_group) == 0) sh.pmax[s][warp][r] = m;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
    }
}

// ----------------------------------------------------------------------------------- 2. Top-k
__global__ void __launch_bounds__(32) decode_topk_kernel(DecodeArgs a, int nb_max)
{
    const int beta = blockIdx.x, r = blockIdx.y, lane = threadIdx.x;
    const int len = a.lens[beta];
    int32_t* sel = a.sel + ((int64_t)beta * a.H_kv + r) * a.k;
    if (len < 1 || len > a.L_max) {
        if (lane == 0) {
            report_error(a.err, MSA_ERR_DEVICE_CHECK, 200 + beta);
            if (r == 0) a.nsel[beta] = 0;
        }
        if (lane < a.k) {
            sel[lane] = -1;
            if (a.block_idx_out) a.block_idx_out[((int64_t)beta * a.H_kv + r) * a.k + lane] = -1;
        }
        return;
    }
    const int local = seq_local_block(len);
    const float* row = a.pooled + ((int64_t)beta * a.H_kv + r) * nb_max;
    TopkList list;
    list.init(a.k - 1);
    for (int b = lane; b < local; b += 32) list.offer_ascending(row[b], b); // each lane: ascending blocks
    float bv[kMaxK - 1];
    int bb[kMaxK - 1];
    warp_merge(list, a.k - 1, bv, bb);
    if (lane == 0) {
        TopkList res;
#pragma unroll
        for (int j = 0; j < TopkList::L; ++j) {
            res.v[j] = bv[j];
            res.b[j] = bb[j];
        }
        int32_t out[kMaxK];
        emit_selection(res, local, a.k, out);
        for (int j = 0; j < a.k; ++j) {
            sel[j] = out[j];
            if (a.block_idx_out) a.block_idx_out[((int64_t)beta * a.H_kv + r) * a.k + j] = out[j];
        }
        if (r == 0) a.nsel[beta] = min(a.k, local + 1);
    }
}

// ----------------------------------------------------------------------------------- 3. attention
template <int DH>
struct DecCfg {
    static constexpr int LD = DH + 8; // padded row (elements): conflict-free fragment loads
    // K, V, Q tiles and the per-warp max / sum; the per-warp outputs [4][16][DH] fp32 reuse the K
    // tile, which no warp reads after S (three CTAs fit per SM)
    static constexpr int SMEM = (2 * 128 * LD + 16 * LD) * 2 + 3 * 4 * 16 * 4;
    static_assert(4 * 16 * DH * 4 <= 128 * LD * 2, "output scratch fits in the K tile");
};

template <int DH>
__global__ void __launch_bounds__(128) decode_attn_kernel(DecodeArgs a)
{
    using C = DecCfg<DH>;
    constexpr int LD = C::LD;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint16_t* sK = reinterpret_cast<uint16_t*>(smem_raw);
    uint16_t* sV = sK + 128 * LD;
    uint16_t* sQ = sV + 128 * LD;
    float* sO = reinterpret_cast<float*>(sK);                  // [4][16][DH], written after S
    float* sMax = reinterpret_cast<float*>(sQ + 16 * LD);     // [4][16]
    float* sSum = sMax + 4 * 16;                               // [4][16] row sums of exp (exact)
    float* sSumR = sSum + 4 * 16;                              // [4][16] row sums of the bf16-rounded P

    const int beta = blockIdx.x, r = blockIdx.y, slot = blockIdx.z;
    const int G = a.H_q / a.H_kv;
    const int b = a.sel[((int64_t)beta * a.H_kv + r) * a.k + slot];
    if (b < 0) return;
    const int len = a.lens[beta];
    const int kv_lim = min(127, len - 1 - b * kBk); // keys 0..kv_lim of the block are visible
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;

    // stage K, V (rows past kv_lim are zero), Q (rows past G are zero)
    const int64_t row_stride = (int64_t)a.H_kv * DH;
    const uint16_t* kb = a.k_cache + (((int64_t)beta * a.L_max + (int64_t)b * kBk) * a.H_kv + r) * DH;
    const uint16_t* vb = a.v_cache + (((int64_t)beta * a.L_max + (int64_t)b * kBk) * a.H_kv + r) * DH;
    constexpr int CPR = DH / 8; // 16-byte chunks per row
    for (int c = tid; c < 128 * CPR; c += 128) {
        const int j = c / CPR, u = c % CPR;
        if (j <= kv_lim) {
            cp_async16(sK + j * LD + u * 8, kb + j * row_stride + u * 8);
            cp_async16(sV + j * LD + u * 8, vb + j * row_stride + u * 8);
        } else {
            *reinterpret_cast<uint4*>(sK + j * LD + u * 8) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(sV + j * LD + u * 8) = make_uint4(0, 0, 0, 0);
        }
    }
    const uint16_t* qb = a.q + ((int64_t)beta * a.H_q + (int64_t)r * G) * DH;
    for (int c = tid; c < 16 * CPR; c += 128) {
        const int j = c / CPR, u = c % CPR;
        if (j < G)
            cp_async16(sQ + j * LD + u * 8, qb + (int64_t)j * DH + u * 8);
        else
            *reinterpret_cast<uint4*>(sQ + j * LD + u * 8) = make_uint4(0, 0, 0, 0);
    }
    cp_async_wait_all();
    __syncthreads();

    // S = Q K^T for keys 32*warp .. +31 (4 n-tiles of 8)
    float sacc[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) sacc[n][q] = 0.f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
        uint32_t af[4];
        const int c0 = ks * 16 + 2 * t;
        af[0] = *reinterpret_cast<const uint32_t*>(sQ + g * LD + c0);
        af[1] = *reinterpret_cast<const uint32_t*>(sQ + (g + 8) * LD + c0);
        af[2] = *reinterpret_cast<const uint32_t*>(sQ + g * LD + c0 + 8);
        af[3] = *reinterpret_cast<const uint32_t*>(sQ + (g + 8) * LD + c0 + 8);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int key = warp * 32 + n * 8 + g;
            const uint32_t b0 = *reinterpret_cast<const uint32_t*>(sK + key * LD + c0);
            const uint32_t b1 = *reinterpret_cast<const uint32_t*>(sK + key * LD + c0 + 8);
            mma_bf16_16816(sacc[n], af, b0, b1);
        }
    }
    // mask, row max (rows g and g+8)
    float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int key = warp * 32 + n * 8 + 2 * t + (q & 1);
            if (key > kv_lim) sacc[n][q] = -CUDART_INF_F;
            if (q < 2)
                mx0 = fmaxf(mx0, sacc[n][q]);
            else
                mx1 = fmaxf(mx1, sacc[n][q]);
        }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (t == 0) {
        sMax[warp * 16 + g] = mx0;
        sMax[warp * 16 + g + 8] = mx1;
    }
    __syncthreads();
    float M0 = -CUDART_INF_F, M1 = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        M0 = fmaxf(M0, sMax[w * 16 + g]);
        M1 = fmaxf(M1, sMax[w * 16 + g + 8]);
    }
    const float scale = rsqrtf((float)DH);
    const float sl2 = scale * 1.4426950408889634f;
    // P = exp(S*scale - M*scale), partial row sums, bf16 A fragments. Two row sums: the exact one
    // gives the lse (the weights the combine merges with); the sum of the bf16-rounded P the PV
    // product uses normalises O, so each partial is an exact weighted average of V rows.
    float l0 = 0.f, l1 = 0.f, lr0 = 0.f, lr1 = 0.f;
    uint32_t pf[2][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const float p0 = ex2_approx(fmaf(sacc[n][0], sl2, -M0 * sl2));
        const float p1 = ex2_approx(fmaf(sacc[n][1], sl2, -M0 * sl2));
        const float p2 = ex2_approx(fmaf(sacc[n][2], sl2, -M1 * sl2));
        const float p3 = ex2_approx(fmaf(sacc[n][3], sl2, -M1 * sl2));
        l0 += p0 + p1;
        l1 += p2 + p3;
        const int kk = n >> 1, hi = n & 1;
        pf[kk][hi * 2 + 0] = pack_bf16x2(p0, p1);
        pf[kk][hi * 2 + 1] = pack_bf16x2(p2, p3);
        lr0 += bf16_lo(pf[kk][hi * 2 + 0]) + bf16_hi(pf[kk][hi * 2 + 0]);
        lr1 += bf16_lo(pf[kk][hi * 2 + 1]) + bf16_hi(pf[kk][hi * 2 + 1]);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        lr0 += __shfl_xor_sync(0xffffffffu, lr0, o);
        lr1 += __shfl_xor_sync(0xffffffffu, lr1, o);
    }
    if (t == 0) {
        sSum[warp * 16 + g] = l0;
        sSum[warp * 16 + g + 8] = l1;
        sSumR[warp * 16 + g] = lr0;
        sSumR[warp * 16 + g + 8] = lr1;
    }
    // O_w = P_w V_w over this warp's 32 keys
    float oacc[DH / 8][4];
#pragma unroll
    for (int n = 0; n < DH / 8; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) oacc[n][q] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        // A fragment order: a0 (row g, keys 2t), a1 (row g+8), a2 (row g, keys 8+2t), a3 (row g+8, 8+2t)
        const uint32_t af[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
        const int key0 = warp * 32 + kk * 16;
#pragma unroll
        for (int n = 0; n < DH / 8; ++n) {
            uint32_t b0, b1;
            const int lr = lane & 15;
            ldmatrix_x2_trans(b0, b1, sV + (key0 + lr) * LD + n * 8);
            mma_bf16_16816(oacc[n], af, b0, b1);
        }
    }
#pragma unroll
    for (int n = 0; n < DH / 8; ++n) {
        const int col = n * 8 + 2 * t;
        sO[(warp * 16 + g) * DH + col] = oacc[n][0];
        sO[(warp * 16 + g) * DH + col + 1] = oacc[n][1];
        sO[(warp * 16 + g + 8) * DH + col] = oacc[n][2];
        sO[(warp * 16 + g + 8) * DH + col + 1] = oacc[n][3];
    }
    __syncthreads();
    // reduce the 4 warps' partials, normalise, write the slot's partial
    for (int e = tid; e < G * DH / 2; e += 128) {
        const int row = (2 * e) / DH, col = (2 * e) % DH;
        float o0 = 0.f, o1 = 0.f, l = 0.f, lr = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            o0 += sO[(w * 16 + row) * DH + col];
            o1 += sO[(w * 16 + row) * DH + col + 1];
            l += sSum[w * 16 + row];
            lr += sSumR[w * 16 + row];
        }
        const float inv = 1.f / lr;
        const int h = r * G + row;
        // partial layout [sequence][slot][d_h/16][H_q][16] (as prefill's stage 1)
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.o_part + ((int64_t)beta * a.k + slot) * a.H_q * DH +
                                                    ((int64_t)(col >> 4) * a.H_q + h) * 16 + (col & 15));
        *dst = pack_bf16x2(o0 * inv, o1 * inv);
        if (col == 0) {
            float Mr = -CUDART_INF_F;
#pragma unroll
            for (int w = 0; w < 4; ++w) Mr = fmaxf(Mr, sMax[w * 16 + row]);
            a.lse_part[((int64_t)beta * a.k + slot) * a.H_q + h] = Mr * scale + logf(l);
        }
    }
}

} // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s)
{
    const int nb_max = (int)((a.L_max + kBk - 1) / kBk);
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (a.H_kv * a.d_idx > 256) return cudaErrorInvalidValue; // a cache row must fit a 512-byte stage row
    cudaError_t e0 = cudaFuncSetAttribute(decode_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPoolSmem);
    if (e0 != cudaSuccess) return e0;
    trace_begin(s);
    decode_prefix_kernel<<<1, 1024, 0, s>>>(a);
    // one CTA per SM, each an equal slice of the flattened block list
    decode_pool_kernel<<<n_sm, (kPoolConsumers + 1) * 32, kPoolSmem, s>>>(a, nb_max);
    trace_end(s, MSA_KERNEL_DEC_POOL);
    trace_begin(s);
    decode_topk_kernel<<<dim3(a.B, a.H_kv), 32, 0, s>>>(a, nb_max);
    trace_end(s, MSA_KERNEL_DEC_TOPK);
    note_launch(4);
    trace_begin(s);
    cudaError_t e;
    if (a.d_h == 128) {
        e = cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DecCfg<128>::SMEM);
        if (e != cudaSuccess) return e;
        decode_attn_kernel<128><<<dim3(a.B, a.H_kv, a.k), 128, DecCfg<128>::SMEM, s>>>(a);
    } else if (a.d_h == 64) {
        e = cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DecCfg<64>::SMEM);
        if (e != cudaSuccess) return e;
        decode_attn_kernel<64><<<dim3(a.B, a.H_kv, a.k), 128, DecCfg<64>::SMEM, s>>>(a);
    } else {
        return cudaErrorInvalidValue;
    }
    trace_end(s, MSA_KERNEL_DEC_ATTN);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CombineArgs c;
    c.row0 = 0;
    c.n_rows = a.B;
    c.H_q = a.H_q;
    c.d_h = a.d_h;
    c.k = a.k;
    c.local_of_row_div = kBk;
    c.o_part = a.o_part;
    c.lse_part = a.lse_part;
    c.nsel = a.nsel;
    c.out = a.out;
    c.lse = a.lse;
    trace_begin(s);
    e = launch_combine(c, s);
    trace_end(s, MSA_KERNEL_DEC_COMBINE);
    return e;
}

} // namespace msa
