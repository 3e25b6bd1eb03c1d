// fp8.cu -- per-row OCP E4M3 quantisation of q, k, v for the FP8 main branch (the "MiniMax M3" blog
// post names FP8 tensor cores for the kernels and gives no quantisation; reading: one scale per
// (token, head) row, scale = amax / 448, codes rounded to nearest with ties to the even code,
// saturating at 448, subnormals kept).
//
// One warp per row of d_h elements: the row's amax by warp shuffles, then every element's code from
// its quotient x / scale computed in fp64 exactly as the definition states (two correctly rounded
// fp64 divisions), so the rounding decision at a code midpoint is the same on every conforming
// implementation. Besides the codes the kernel writes the row scales and their reciprocals in a
// head-major layout [H][S] (S = N rounded up to whole 128-token blocks, padding tokens get scale 1 so
// that every block's scale run is finite and 512 bytes long), and optionally the largest scale of
// every (head, 128-token block), which the attention uses to keep the FP8 P' = P * s_v in range.
#include "common.cuh"

namespace msa {

namespace {

// Nearest E4M3 code of q (ties to the even code; |q| >= 448 saturates to 448; NaN cannot occur here).
__device__ __forceinline__ uint8_t e4m3_encode_rne(double q)
{
    const uint8_t sign = signbit(q) ? 0x80 : 0;
    const double a = fabs(q);
    if (!(a < 448.0)) return sign | 0x7E;
    if (a < 0.015625) // below 2^-6: subnormal codes, step 2^-9 (8 * 2^-9 = 2^-6 is the first normal code)
        return sign | (uint8_t)rint(a * 512.0);
    int e = 0;
    const double f = frexp(a, &e); // a = f * 2^e, f in [0.5, 1): a = (n / 8) * 2^(e-1), n in [8, 16)
    int n = (int)rint(ldexp(f, 4));
    int E = e - 1;
    if (n == 16) {
        n = 8;
        ++E;
    }
    return sign | (uint8_t)(((E + 7) << 3) | (n - 8));
}

__global__ void quantize_e4m3_kernel(QuantArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t nrows = a.N * a.H;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    constexpr int kMaxPer = 8; // d <= 256
    const int per = a.d / 32;
    for (int64_t row = warp0; row < a.N_pad * a.H; row += nwarps) {
        const int64_t n = row / a.H;
        const int h = (int)(row - n * a.H);
        float x[kMaxPer];
        float amax = 0.f;
        if (row < nrows) {
            const uint16_t* src = a.x + row * a.d + lane * per;
#pragma unroll
            for (int i = 0; i < kMaxPer; ++i)
                if (i < per) {
                    x[i] = __uint_as_float((uint32_t)src[i] << 16);
                    amax = fmaxf(amax, fabsf(x[i]));
                }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const double scale = amax > 0.f ? (double)amax / 448.0 : 1.0;
        if (row < nrows) {
            uint8_t* dst = a.codes + row * a.d + lane * per;
#pragma unroll
            for (int i = 0; i < kMaxPer; ++i)
                if (i < per) dst[i] = e4m3_encode_rne((double)x[i] / scale);
        }
        if (lane == 0) {
            const float s32 = (float)scale;
            a.scales[(int64_t)h * a.N_pad + n] = s32;
            if (a.rscales) a.rscales[(int64_t)h * a.N_pad + n] = (float)(1.0 / scale);
            // scales are positive: their bit patterns order like the values
            if (a.blkmax && row < nrows)
                atomicMax(reinterpret_cast<int*>(a.blkmax) + (int64_t)h * a.nb + n / kBk, __float_as_int(s32));
        }
    }
}

} // namespace

cudaError_t launch_quantize_e4m3(const QuantArgs& a, cudaStream_t s)
{
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows = a.N_pad * a.H;
    const int64_t want = (rows + 7) / 8; // 8 warps per CTA
    const int grid = (int)(want < (int64_t)n_sm * 16 ? want : (int64_t)n_sm * 16);
    quantize_e4m3_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(a);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace msa
