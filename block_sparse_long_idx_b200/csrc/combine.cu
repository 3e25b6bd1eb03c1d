// combine.cu -- stage 2 of the two-stage forward: split-K merge of the per-block partials through
// their log-sum-exp ("MiniMax Sparse Attention" explainer, section 05-2: the attention kernel writes
// each query's k partials into preallocated slots and a combine kernel merges them via the LSE; the
// LSE is also written out for the sparse-KL backward).
//
// For row i and head h with valid slots s < n_sel(i):
//   M = max_s lse_s,  w_s = exp(lse_s - M),  L = sum_s w_s
//   out[i, h] = sum_s (w_s / L) * o_s,        lse[i, h] = M + log(L)
// Slots are merged in the fixed order 0..n_sel-1, so the result is deterministic.
//
// Partials are laid out [row][slot][d_h/16][H_q][16] (bf16) and [row][slot][H_q] (fp32 lse). One CTA
// per row reads the row's contiguous slabs with 16-byte loads (all slots of a unit in flight at
// once), and stages the merged row in shared memory so the output row is written contiguously.
#include <math_constants.h>

#include "common.cuh"

namespace msa {

namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a)
{
    extern __shared__ __align__(16) uint8_t csm[];
    float* wsm = reinterpret_cast<float*>(csm);                                 // [k][H_q] weights
    uint4* obuf = reinterpret_cast<uint4*>(csm + align_up_dev(a.k * a.H_q * 4)); // [H_q][d_h/8] swizzled
    const int64_t i = a.row0 + blockIdx.x;
    const int64_t prow = blockIdx.x;
    const int64_t il = a.row_start ? i - a.row_start[i] : i; // row index within its sequence
    const int n_sel = a.nsel ? a.nsel[prow] : (int)min((int64_t)a.k, il / a.local_of_row_div + 1);
    if (n_sel <= 0) return; // rejected decode sequence: output left unwritten
    const float* lp = a.lse_part + prow * a.k * a.H_q;
    for (int h = threadIdx.x; h < a.H_q; h += blockDim.x) {
        float M = -CUDART_INF_F;
        for (int s = 0; s < n_sel; ++s) M = fmaxf(M, lp[s * a.H_q + h]);
        float L = 0.f;
        for (int s = 0; s < n_sel; ++s) {
            const float w = expf(lp[s * a.H_q + h] - M);
            wsm[s * a.H_q + h] = w;
            L += w;
        }
        const float inv = 1.f / L;
        for (int s = 0; s < n_sel; ++s) wsm[s * a.H_q + h] *= inv;
        if (a.lse) a.lse[i * a.H_q + h] = M + logf(L);
    }
    __syncthreads();
    const int NC = a.d_h / 8;     // 16-byte units per head
    const int units = a.H_q * NC; // per slot
    const uint4* op = reinterpret_cast<const uint4*>(a.o_part + prow * a.k * a.H_q * (int64_t)a.d_h);
    for (int u = threadIdx.x; u < units; u += blockDim.x) {
        // 16-byte unit u of a slot in memory order: 32-byte unit u / (2 H_q), head (u / 2) % H_q, half u % 2
        const int c2 = u / (2 * a.H_q), rem = u - c2 * 2 * a.H_q;
        const int h = rem >> 1, c = 2 * c2 + (rem & 1);
        uint4 v[kMaxK];
#pragma unroll
        for (int s = 0; s < kMaxK; ++s)
            if (s < n_sel) v[s] = op[(int64_t)s * units + u];
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int s = 0; s < kMaxK; ++s) {
            if (s < n_sel) {
                const float w = wsm[s * a.H_q + h];
                const uint32_t x[4] = {v[s].x, v[s].y, v[s].z, v[s].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] = fmaf(w, __uint_as_float(x[q] << 16), acc[2 * q]);
                    acc[2 * q + 1] = fmaf(w, __uint_as_float(x[q] & 0xFFFF0000u), acc[2 * q + 1]);
                }
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t r;
            asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(acc[2 * q]), "f"(acc[2 * q + 1]));
            o[q] = r;
        }
        obuf[h * NC + (c ^ (h & (NC - 1)))] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(a.out + i * a.H_q * (int64_t)a.d_h);
    for (int u = threadIdx.x; u < units; u += blockDim.x) {
        const int h = u / NC, c = u - h * NC;
        dst[u] = obuf[h * NC + (c ^ (h & (NC - 1)))];
    }
}

} // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s)
{
    if (a.n_rows <= 0) return cudaSuccess;
    const size_t smem = align_up((size_t)a.k * a.H_q * sizeof(float), 16) + (size_t)a.H_q * a.d_h * 2;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    combine_kernel<<<(unsigned)a.n_rows, kCombineThreads, smem, s>>>(a);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace msa
