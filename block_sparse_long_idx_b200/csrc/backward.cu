// backward.cu -- gradient of the main branch in q, k and v, with the selected sets held fixed
// ("MiniMax Sparse Attention" explainer, section 03: the Top-k is not differentiable, so the
// language-model loss reaches the main branch only through the exact attention over the selected
// blocks; section 05-2, "LSE fusion" paragraph: the forward's per-head LSE is read back by the
// backward instead of recomputing the softmax normaliser).
//
// For one (row i, head h) with p_j = exp(q.k_j * scale - lse) over its token set T:
//   D = dout . out,   ds_j = p_j (dout . v_j - D),
//   dq_i = scale sum_j ds_j k_j,   dk_j += scale ds_j q_i,   dv_j += p_j dout_i.
//
// KV-outer over the forward's work items (group r, block b, a chunk of the rows that selected b),
// claimed from an atomic counter by a persistent grid. The CTA stages K_b and V_b once and walks
// the item's rows in tiles of 16 (16/G positions x G heads). Warp w owns keys 16w .. 16w+15 of the
// block and keeps their dK and dV in registers for the whole item (mma.sync m16n8k16, fp32
// accumulation):
//   S^T = K_w Q^T,  P^T = exp2(S^T scale log2e - lse log2e)  (0 past the query on its own block),
//   dP^T = V_w dO^T,  dS^T = P^T (dP^T - D),  dV_w += P^T dO,  dK_w += dS^T Q.
// dS^T goes to shared memory as dS (rows x keys); the 8 warps then form the tile's dQ = dS K, one
// d_h/8-column slice each, and add it to the fp32 dq accumulator. At the end of the item dK and
// dV are added to their fp32 accumulators (a hot block's rows are split over several items).
// A last kernel rounds the three accumulators to bf16.
//
// Index-branch KL alignment (explainer section 03, "KL Loss"), optional and fused into the same
// pass: for row i and group r over T(i, r) the student is the softmax of the unscaled index scores
// s_j = q_idx[i,r] . k_idx[j,r], the teacher P_j the average of the group's G attention weights,
// and KL(i, r) = sum_j P_j (log P_j - log P_idx_j); the teacher is stop-gradient, so
//   dq_idx[i,r] += w sum_j (P_idx_j - P_j) k_idx[j,r],   dk_idx[j,r] += w (P_idx_j - P_j) q_idx[i,r].
// A pre-pass gives each (i, r) the log-sum-exp of its index scores over T; in the KV-outer pass the
// teacher of a position is the mean of its G rows of the P^T tile the gradient already computes,
// and the block's k_idx rows and dk_idx accumulators stay in shared memory for the whole item.
#include <math_constants.h>

#include "backward.cuh"
#include "common.cuh"
#include "mma_sync.cuh"

namespace msa {

namespace {

constexpr int kBwdWarps = 8; // 8 x 16 keys = one 128-key block
constexpr int kTileRows = 16;
constexpr float kLog2e = 1.4426950408889634f;

template <int DH, int DI = 0>
struct BwdCfg {
    static constexpr int LD = DH + 8;   // padded row of K, V, Q, dO (elements): conflict-free fragments
    static constexpr int LDS = kBk + 8; // padded row of dS (elements)
    static constexpr int BASE = (2 * kBk * LD + 2 * kTileRows * LD + kTileRows * LDS) * 2 + 3 * kTileRows * 4;
    // KL part (fp32): k_idx block and its dk_idx accumulators [128][DI+1], P^T [16][129], the
    // student-minus-teacher weights [16][128], the tile's q_idx rows [16][DI] and their lse [16]
    static constexpr int LDI = DI + 1;
    static constexpr int LDP = kBk + 1;
    static constexpr int KL = DI ? (2 * kBk * LDI + kTileRows * LDP + kTileRows * kBk + kTileRows * DI + kTileRows) * 4 : 0;
    static constexpr int SMEM = BASE + KL;
    static_assert(BASE % 16 == 0, "KL region alignment");
};

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// D[i, h] = dout[i, h, :] . out[i, h, :], one warp per (row, head)
template <int DH>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdArgs a)
{
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= a.N * a.H_q) return;
    constexpr int PER = DH / 32;
    const uint16_t* o = a.out + w * DH + lane * PER;
    const uint16_t* g = a.dout + w * DH + lane * PER;
    float acc = 0.f;
    if constexpr (PER == 4) {
        const uint2 x = *reinterpret_cast<const uint2*>(o);
        const uint2 y = *reinterpret_cast<const uint2*>(g);
        acc = bf_lo(x.x) * bf_lo(y.x) + bf_hi(x.x) * bf_hi(y.x) + bf_lo(x.y) * bf_lo(y.y) + bf_hi(x.y) * bf_hi(y.y);
    } else {
        const uint32_t x = *reinterpret_cast<const uint32_t*>(o);
        const uint32_t y = *reinterpret_cast<const uint32_t*>(g);
        acc = bf_lo(x) * bf_lo(y) + bf_hi(x) * bf_hi(y);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) a.D[w] = acc;
}

// log-sum-exp of the unscaled index scores of (i, r) over T(i, r), one warp per (i, r); each lane
// scores whole keys (lane + 32u of every selected block) and keeps an online (max, sum)
template <int DI>
__global__ void __launch_bounds__(256) kl_lse_kernel(BwdArgs a)
{
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; // (i, r) = (w / H_kv, w % H_kv)
    const int lane = threadIdx.x & 31;
    if (w >= a.N * a.H_kv) return;
    const int64_t i = w / a.H_kv;
    const int r = (int)(w % a.H_kv);
    float q[DI];
    const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q_idx + w * DI);
#pragma unroll
    for (int d = 0; d < DI / 2; ++d) {
        const uint32_t u = qp[d];
        q[2 * d] = bf_lo(u);
        q[2 * d + 1] = bf_hi(u);
    }
    float m = -CUDART_INF_F, l = 0.f;
    const int32_t* sel = a.block_idx + ((int64_t)r * a.N + i) * a.k;
    for (int s = 0; s < a.k; ++s) {
        const int32_t b = sel[s];
        if (b < 0 || (int64_t)b * kBk > i) continue;
#pragma unroll
        for (int u = 0; u < kBk / 32; ++u) {
            const int64_t j = (int64_t)b * kBk + lane + 32 * u;
            if (j > i) continue;
            const uint4* kp = reinterpret_cast<const uint4*>(a.k_idx + (j * a.H_kv + r) * DI);
            float sdot = 0.f;
#pragma unroll
            for (int c = 0; c < DI / 8; ++c) {
                const uint4 x = kp[c];
                sdot = fmaf(q[8 * c + 0], bf_lo(x.x), sdot);
                sdot = fmaf(q[8 * c + 1], bf_hi(x.x), sdot);
                sdot = fmaf(q[8 * c + 2], bf_lo(x.y), sdot);
                sdot = fmaf(q[8 * c + 3], bf_hi(x.y), sdot);
                sdot = fmaf(q[8 * c + 4], bf_lo(x.z), sdot);
                sdot = fmaf(q[8 * c + 5], bf_hi(x.z), sdot);
                sdot = fmaf(q[8 * c + 6], bf_lo(x.w), sdot);
                sdot = fmaf(q[8 * c + 7], bf_hi(x.w), sdot);
            }
            if (sdot > m) {
                l = l * expf(m - sdot) + 1.f;
                m = sdot;
            } else {
                l += expf(sdot - m);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float M = fmaxf(m, m2);
        l = (m == -CUDART_INF_F ? 0.f : l * expf(m - M)) + (m2 == -CUDART_INF_F ? 0.f : l2 * expf(m2 - M));
        m = M;
    }
    if (lane == 0) a.lse_idx[w] = m + logf(l);
}

template <int DH, int G, int DI>
__global__ void __launch_bounds__(kBwdWarps * 32, 1) bwd_attn_kernel(BwdArgs a)
{
    using C = BwdCfg<DH, DI>;
    constexpr int LD = C::LD, LDS = C::LDS;
    constexpr int PPT = kTileRows / G; // positions per tile
    constexpr int CPR = DH / 8;        // 16-byte chunks per row
    constexpr int NQT = DH / 64;       // 8-column n-tiles of each warp's dQ slice
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint16_t* sK = reinterpret_cast<uint16_t*>(smem_raw);
    uint16_t* sV = sK + kBk * LD;
    uint16_t* sQ = sV + kBk * LD;
    uint16_t* sdO = sQ + kTileRows * LD;
    uint16_t* sdS = sdO + kTileRows * LD;
    float* sLse = reinterpret_cast<float*>(sdS + kTileRows * LDS); // lse * log2e (+inf: no row)
    float* sD = sLse + kTileRows;
    int* sPos = reinterpret_cast<int*>(sD + kTileRows); // query position of each tile row (-1: none)
    // KL part (unused when DI == 0)
    constexpr int LDI = C::LDI, LDP = C::LDP;
    float* sKI = reinterpret_cast<float*>(smem_raw + C::BASE); // [128][LDI] k_idx of the block
    float* sDKI = sKI + kBk * LDI;                             // [128][LDI] dk_idx of the block
    float* sP = sDKI + kBk * LDI;                              // [16][LDP] P^T of the tile (row-major)
    float* sG = sP + kTileRows * LDP;                          // [PPT][128] w (P_idx - P) per position, key
    float* sQI = sG + kTileRows * kBk;                         // [PPT][DI] q_idx of the tile's positions
    float* sLI = sQI + kTileRows * (DI > 0 ? DI : 1);           // [PPT] lse of the index scores
    __shared__ int s_item;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3, lr = lane & 15;
    const int kw0 = warp * 16;
    const int64_t Nk = a.N * a.k;
    const int64_t kv_stride = (int64_t)a.H_kv * DH;
    const int n_items = a.window_items[a.n_windows];
    const float scale = rsqrtf((float)DH);
    const float sl2 = scale * kLog2e;

    for (;;) {
        __syncthreads(); // every thread has read s_item and finished with the previous item's tiles
        if (tid == 0) s_item = atomicAdd(a.item_counter, 1);
        __syncthreads();
        const int j = s_item;
        if (j >= n_items) break;
        const msa_work_item it = a.items[j];
        const int r = it.r;
        const int64_t tok0 = (int64_t)it.b * kBk;
        if (r < 0 || r >= a.H_kv || tok0 >= a.N || it.len < 0) {
            if (tid == 0) report_error(a.err, MSA_ERR_DEVICE_CHECK, 400);
            continue;
        }
        // stage K_b and V_b (rows past N are zero)
        const uint16_t* kb = a.kk + (tok0 * a.H_kv + r) * DH;
        const uint16_t* vb = a.v + (tok0 * a.H_kv + r) * DH;
        for (int c = tid; c < kBk * CPR; c += kBwdWarps * 32) {
            const int jj = c / CPR, u = c % CPR;
            if (tok0 + jj < a.N) {
                cp_async16(sK + jj * LD + u * 8, kb + jj * kv_stride + u * 8);
                cp_async16(sV + jj * LD + u * 8, vb + jj * kv_stride + u * 8);
            } else {
                *reinterpret_cast<uint4*>(sK + jj * LD + u * 8) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sV + jj * LD + u * 8) = make_uint4(0, 0, 0, 0);
            }
        }
        if constexpr (DI > 0) {
            for (int c = tid; c < kBk * DI; c += kBwdWarps * 32) {
                const int jj = c / DI, d = c % DI;
                float x = 0.f;
                if (tok0 + jj < a.N) {
                    const uint16_t u = a.k_idx[((tok0 + jj) * a.H_kv + r) * DI + d];
                    x = __uint_as_float((uint32_t)u << 16);
                }
                sKI[jj * LDI + d] = x;
                sDKI[jj * LDI + d] = 0.f;
            }
        }
        float dk[DH / 8][4], dv[DH / 8][4];
#pragma unroll
        for (int n = 0; n < DH / 8; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) dk[n][q] = dv[n][q] = 0.f;

        const int ntiles = (it.len + PPT - 1) / PPT;
        for (int tile = 0; tile < ntiles; ++tile) {
            // tile row = position pl * G + head hh
            if (tid < kTileRows) {
                const int row = tid, pl = row / G, hh = row % G;
                const int idx = tile * PPT + pl;
                int pos = -1;
                if (idx < it.len) {
                    const int32_t e = a.entries[(int64_t)r * Nk + it.start + idx];
                    const int p = e / a.k;
                    if (e < 0 || p >= a.N)
                        report_error(a.err, MSA_ERR_DEVICE_CHECK, 401);
                    else
                        pos = p;
                }
                sPos[row] = pos;
                const int64_t rh = (int64_t)pos * a.H_q + r * G + hh;
                sLse[row] = pos >= 0 ? a.lse[rh] * kLog2e : CUDART_INF_F;
                sD[row] = pos >= 0 ? a.D[rh] : 0.f;
            }
            __syncthreads();
            for (int c = tid; c < kTileRows * CPR; c += kBwdWarps * 32) {
                const int row = c / CPR, u = c % CPR;
                const int pos = sPos[row];
                if (pos >= 0) {
                    const int64_t off = ((int64_t)pos * a.H_q + r * G + row % G) * DH + u * 8;
                    cp_async16(sQ + row * LD + u * 8, a.q + off);
                    cp_async16(sdO + row * LD + u * 8, a.dout + off);
                } else {
                    *reinterpret_cast<uint4*>(sQ + row * LD + u * 8) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sdO + row * LD + u * 8) = make_uint4(0, 0, 0, 0);
                }
            }
            if constexpr (DI > 0) {
                for (int c = tid; c < PPT * DI; c += kBwdWarps * 32) {
                    const int pl = c / DI, d = c % DI;
                    const int pos = sPos[pl * G];
                    sQI[c] = pos >= 0 ? __uint_as_float((uint32_t)a.q_idx[((int64_t)pos * a.H_kv + r) * DI + d] << 16)
                                      : 0.f;
                }
                if (tid < PPT) {
                    const int pos = sPos[tid * G];
                    sLI[tid] = pos >= 0 ? a.lse_idx[(int64_t)pos * a.H_kv + r] : 0.f;
                }
            }
            cp_async_wait_all();
            __syncthreads();

            // S^T = K_w Q^T and dP^T = V_w dO^T: keys kw0 .. kw0+15 x the 16 rows (two n-tiles). A
            // fragments (K_w, V_w rows) and the B fragments of both n-tiles (Q, dO rows) by ldmatrix.x4:
            // B matrices are (rows 0-7, d 0-7), (rows 0-7, d 8-15), (rows 8-15, d 0-7), (rows 8-15, d 8-15)
            float st[2][4], dpt[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) st[n][q] = dpt[n][q] = 0.f;
            const int a_off = (kw0 + (lane & 15)) * LD + (lane >> 4) * 8;
            const int b_off = ((lane & 7) + ((lane >> 4) << 3)) * LD + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < DH / 16; ++ks) {
                uint32_t ak[4], av[4], bq[4], bo[4];
                ldmatrix_x4(ak[0], ak[1], ak[2], ak[3], sK + a_off + ks * 16);
                ldmatrix_x4(av[0], av[1], av[2], av[3], sV + a_off + ks * 16);
                ldmatrix_x4(bq[0], bq[1], bq[2], bq[3], sQ + b_off + ks * 16);
                ldmatrix_x4(bo[0], bo[1], bo[2], bo[3], sdO + b_off + ks * 16);
                mma_bf16_16816(st[0], ak, bq[0], bq[1]);
                mma_bf16_16816(st[1], ak, bq[2], bq[3]);
                mma_bf16_16816(dpt[0], av, bo[0], bo[1]);
                mma_bf16_16816(dpt[1], av, bo[2], bo[3]);
            }
            // P^T and dS^T; element (n, q) is key kw0 + g (+8 for q >= 2), row n*8 + 2t + (q & 1)
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = kw0 + g + ((q & 2) ? 8 : 0);
                    const int row = n * 8 + 2 * t + (q & 1);
                    const int pos = sPos[row];
                    float p = ex2_approx(fmaf(st[n][q], sl2, -sLse[row]));
                    if (pos < 0 || tok0 + key > pos) p = 0.f; // causal on the query's own block
                    st[n][q] = p;
                    dpt[n][q] = p * (dpt[n][q] - sD[row]);
                }
            // A fragments (keys x rows): a0 (key g, rows 2t), a1 (key g+8), a2 (key g, rows 8+2t), a3
            const uint32_t pa[4] = {pack_bf16x2(st[0][0], st[0][1]), pack_bf16x2(st[0][2], st[0][3]),
                                    pack_bf16x2(st[1][0], st[1][1]), pack_bf16x2(st[1][2], st[1][3])};
            const uint32_t da[4] = {pack_bf16x2(dpt[0][0], dpt[0][1]), pack_bf16x2(dpt[0][2], dpt[0][3]),
                                    pack_bf16x2(dpt[1][0], dpt[1][1]), pack_bf16x2(dpt[1][2], dpt[1][3])};
            // dV_w += P^T dO, dK_w += dS^T Q (the 16 rows are the contraction)
#pragma unroll
            for (int n = 0; n < DH / 8; ++n) {
                uint32_t b0, b1;
                ldmatrix_x2_trans(b0, b1, sdO + lr * LD + n * 8);
                mma_bf16_16816(dv[n], pa, b0, b1);
                ldmatrix_x2_trans(b0, b1, sQ + lr * LD + n * 8);
                mma_bf16_16816(dk[n], da, b0, b1);
            }
            // dS (rows x keys) to shared memory, rounded like the operand of the dK product
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = kw0 + g + ((q & 2) ? 8 : 0);
                    const int row = n * 8 + 2 * t + (q & 1);
                    sdS[row * LDS + key] = (uint16_t)(pack_bf16x2(dpt[n][q], 0.f) & 0xffffu);
                    if constexpr (DI > 0) sP[row * LDP + key] = st[n][q];
                }
            __syncthreads();
            // dQ of the tile, columns warp*DH/8 .. +DH/8: dS (16 x 128 keys) K (128 keys x DH)
            float dq[NQT][4];
#pragma unroll
            for (int n = 0; n < NQT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) dq[n][q] = 0.f;
#pragma unroll
            for (int ks = 0; ks < kBk / 16; ++ks) {
                uint32_t af[4];
                ldmatrix_x4(af[0], af[1], af[2], af[3], sdS + (lane & 15) * LDS + (lane >> 4) * 8 + ks * 16);
#pragma unroll
                for (int n = 0; n < NQT; ++n) {
                    uint32_t b0, b1;
                    ldmatrix_x2_trans(b0, b1, sK + (ks * 16 + lr) * LD + warp * (DH / 8) + n * 8);
                    mma_bf16_16816(dq[n], af, b0, b1);
                }
            }
#pragma unroll
            for (int n = 0; n < NQT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = g + ((q & 2) ? 8 : 0);
                    const int col = warp * (DH / 8) + n * 8 + 2 * t + (q & 1);
                    const int pos = sPos[row];
                    if (pos >= 0)
                        atomicAdd(a.dq_acc + ((int64_t)pos * a.H_q + r * G + row % G) * DH + col, scale * dq[n][q]);
                }
            if constexpr (DI > 0) {
                // per (position, key): teacher = mean of the position's G rows of P^T, student weight
                // from the index score; thread = (key j, half of the d_idx dimensions)
                const int j = tid & (kBk - 1), half = tid >> 7;
                const int64_t key = tok0 + j;
                for (int pl = 0; pl < PPT; ++pl) {
                    const int pos = sPos[pl * G];
                    const bool valid = pos >= 0 && key <= pos;
                    float T = 0.f;
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) T += sP[(pl * G + hh) * LDP + j];
                    T *= 1.f / G;
                    float sidx = 0.f;
#pragma unroll 8
                    for (int d = 0; d < DI; ++d) sidx = fmaf(sQI[pl * DI + d], sKI[j * LDI + d], sidx);
                    const float lq = sidx - sLI[pl]; // log of the student weight
                    const float gw = valid ? a.kl_weight * (expf(lq) - T) : 0.f;
                    if (half == 0) sG[pl * kBk + j] = gw;
#pragma unroll 8
                    for (int d = half * (DI / 2); d < (half + 1) * (DI / 2); ++d)
                        sDKI[j * LDI + d] = fmaf(gw, sQI[pl * DI + d], sDKI[j * LDI + d]);
                    if (a.kl != nullptr && half == 0) { // warp-uniform
                        float term = (valid && T > 0.f) ? T * (logf(T) - lq) : 0.f;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
                        if (lane == 0 && pos >= 0) atomicAdd(a.kl + (int64_t)pos * a.H_kv + r, term);
                    }
                }
                __syncthreads();
                // dq_idx of each position: sum over the block's keys of w (P_idx - P) k_idx, each output
                // split over PARTS key ranges so that all threads share the work
                constexpr int OUT = PPT * DI;
                constexpr int PARTS = OUT >= kBwdWarps * 32 ? 1 : kBwdWarps * 32 / OUT;
                constexpr int KPP = kBk / PARTS;
                static_assert(kBk % PARTS == 0, "key ranges");
                for (int c = tid; c < OUT * PARTS; c += kBwdWarps * 32) {
                    const int o = c % OUT, part = c / OUT;
                    const int pl = o / DI, d = o % DI;
                    const int pos = sPos[pl * G];
                    if (pos < 0) continue;
                    float acc = 0.f;
#pragma unroll 8
                    for (int jj = part * KPP; jj < (part + 1) * KPP; ++jj)
                        acc = fmaf(sG[pl * kBk + jj], sKI[jj * LDI + d], acc);
                    atomicAdd(a.dqi_acc + ((int64_t)pos * a.H_kv + r) * DI + d, acc);
                }
            }
            __syncthreads(); // sQ, sdO, sdS and the row tables are free for the next tile
        }
        cp_async_wait_all(); // an item without rows still has its K/V copies in flight
        if constexpr (DI > 0) {
            __syncthreads(); // every thread's dk_idx updates (or, without rows, the zeroing) are visible
            for (int c = tid; c < kBk * DI; c += kBwdWarps * 32) {
                const int jj = c / DI, d = c % DI;
                if (tok0 + jj < a.N) atomicAdd(a.dki_acc + ((tok0 + jj) * a.H_kv + r) * DI + d, sDKI[jj * LDI + d]);
            }
        }
        // the warp's keys: dK and dV into the fp32 accumulators
#pragma unroll
        for (int n = 0; n < DH / 8; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t key = tok0 + kw0 + g + ((q & 2) ? 8 : 0);
                const int col = n * 8 + 2 * t + (q & 1);
                if (key < a.N) {
                    const int64_t off = (key * a.H_kv + r) * DH + col;
                    atomicAdd(a.dk_acc + off, scale * dk[n][q]);
                    atomicAdd(a.dv_acc + off, dv[n][q]);
                }
            }
    }
}

// fp32 accumulators -> bf16 gradients (n4 groups of four values)
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst,
                                                         int64_t n4)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 x = reinterpret_cast<const float4*>(src)[i];
        reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
    }
}

template <int DH, int G, int DI>
cudaError_t launch_attn_cfg(const BwdArgs& a, cudaStream_t s, int n_sm)
{
    const int smem = BwdCfg<DH, DI>::SMEM;
    static_assert(BwdCfg<DH, DI>::SMEM <= 227 * 1024, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(bwd_attn_kernel<DH, G, DI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bwd_attn_kernel<DH, G, DI>, kBwdWarps * 32, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    bwd_attn_kernel<DH, G, DI><<<n_sm * per_sm, kBwdWarps * 32, smem, s>>>(a);
    note_launch(1);
    return cudaGetLastError();
}

template <int DH, int DI>
cudaError_t launch_attn_g(const BwdArgs& a, int G, cudaStream_t s, int n_sm)
{
    switch (G) {
    case 1: return launch_attn_cfg<DH, 1, DI>(a, s, n_sm);
    case 2: return launch_attn_cfg<DH, 2, DI>(a, s, n_sm);
    case 4: return launch_attn_cfg<DH, 4, DI>(a, s, n_sm);
    case 8: return launch_attn_cfg<DH, 8, DI>(a, s, n_sm);
    case 16: return launch_attn_cfg<DH, 16, DI>(a, s, n_sm);
    default: return cudaErrorInvalidValue;
    }
}

template <int DH>
cudaError_t launch_attn_dh(const BwdArgs& a, int G, cudaStream_t s, int n_sm)
{
    if (a.q_idx == nullptr) return launch_attn_g<DH, 0>(a, G, s, n_sm);
    if (a.d_idx == 32) return launch_attn_g<DH, 32>(a, G, s, n_sm);
    if (a.d_idx == 64) return launch_attn_g<DH, 64>(a, G, s, n_sm);
    return cudaErrorInvalidValue;
}

cudaError_t launch_convert(const float* src, uint16_t* dst, int64_t n, cudaStream_t s, int n_sm)
{
    const int64_t n4 = n / 4;
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > (int64_t)n_sm * 8) blocks = (int64_t)n_sm * 8;
    if (blocks < 1) blocks = 1;
    bwd_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, dst, n4);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s)
{
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int G = a.H_q / a.H_kv;
    const int64_t warps = a.N * a.H_q;

    trace_begin(s);
    if (a.d_h == 128)
        bwd_prep_kernel<128><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(a);
    else
        bwd_prep_kernel<64><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(a);
    note_launch(1);
    if (a.q_idx != nullptr) {
        const int64_t wk = a.N * a.H_kv;
        if (a.d_idx == 64)
            kl_lse_kernel<64><<<(unsigned)((wk + 7) / 8), 256, 0, s>>>(a);
        else
            kl_lse_kernel<32><<<(unsigned)((wk + 7) / 8), 256, 0, s>>>(a);
        note_launch(1);
    }
    trace_end(s, MSA_KERNEL_BWD_PREP);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    trace_begin(s);
    e = a.d_h == 128 ? launch_attn_dh<128>(a, G, s, n_sm) : launch_attn_dh<64>(a, G, s, n_sm);
    trace_end(s, MSA_KERNEL_BWD_ATTN);
    if (e != cudaSuccess) return e;

    trace_begin(s);
    e = launch_convert(a.dq_acc, a.dq, a.N * a.H_q * a.d_h, s, n_sm);
    if (e == cudaSuccess) e = launch_convert(a.dk_acc, a.dk, a.N * a.H_kv * a.d_h, s, n_sm);
    if (e == cudaSuccess) e = launch_convert(a.dv_acc, a.dv, a.N * a.H_kv * a.d_h, s, n_sm);
    if (e == cudaSuccess && a.q_idx != nullptr) {
        e = launch_convert(a.dqi_acc, a.dq_idx, a.N * a.H_kv * a.d_idx, s, n_sm);
        if (e == cudaSuccess) e = launch_convert(a.dki_acc, a.dk_idx, a.N * a.H_kv * a.d_idx, s, n_sm);
    }
    trace_end(s, MSA_KERNEL_BWD_CONVERT);
    return e;
}

} // namespace msa
