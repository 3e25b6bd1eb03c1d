// fp8.cu -- per-row OCP E4M3 quantisation of q, k, v for the FP8 main branch (the "MiniMax M3" blog
// post names FP8 tensor cores for the kernels and gives no quantisation; reading: one scale per
// (token, head) row, scale = amax / 448, codes rounded to nearest with ties to the even code,
// saturating at 448, subnormals kept).
//
// One warp per row of d_h elements: the row's amax by warp shuffles, then every element's code. The
// code is decided in fp32 with the hardware E4M3 conversion when the fp32 quotient is clearly away
// from a code midpoint, and otherwise from the quotient x / scale computed in fp64 exactly as the
// definition states (two correctly rounded fp64 divisions), so every code equals the definition's.
// Besides the codes the kernel writes the row scales and their reciprocals in a head-major layout [H][S] (S = N rounded up to whole 128-token blocks, padding tokens get scale 1 so
// that every block's scale run is finite and 512 bytes long), and optionally the largest scale of
// every (head, 128-token block), which the attention uses to keep the FP8 P' = P * s_v in range.
#include "common.cuh"
#include "sm100.cuh"

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

// Code of x / scale with r = 448 / amax in fp32: the fp32 quotient x * r is within 2^-23 (relative)
// of the exact one, i.e. within 2 units of the 20 mantissa bits E4M3 drops; unless it lies within 8
// such units of a code midpoint (or of a subnormal-step midpoint), the hardware conversion (round to
// nearest even, saturating) gives the exact code; otherwise the fp64 quotient x / (amax / 448), the
// definition's, decides.
__device__ __forceinline__ uint8_t e4m3_code(float x, float r, float amax)
{
    const float q = x * r;
    const float a = fabsf(q);
    if (!(r < 3.0e38f)) // amax below ~1.3e-36: 448 / amax overflows fp32, the fp64 quotient is finite
        return e4m3_encode_rne((double)x / ((double)amax / 448.0));
    bool near;
    if (a >= 0.015625f) {
        const uint32_t rem = __float_as_uint(a) & 0xFFFFFu;
        near = rem > 0x80000u - 8u && rem < 0x80000u + 8u;
    } else {
        const float t = a * 512.f; // exact: the subnormal grid in units of 2^-9
        near = fabsf(t - floorf(t) - 0.5f) < 1.0e-4f;
    }
    if (near) return e4m3_encode_rne((double)x / ((double)amax / 448.0));
    return (uint8_t)(e4m3x2_pack(q, 0.f) & 0xFFu);
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
        const int n = (int)((uint32_t)row / (uint32_t)a.H); // N_pad * H < 2^31
        const int h = (int)(row - (int64_t)n * a.H);
        float x[kMaxPer];
        float amax = 0.f;
        if (row < nrows) {
            const uint16_t* src = a.x + row * a.d + lane * per;
            if (per == 4) { // one 8-byte load per lane (the row is 256 bytes, 16-byte aligned)
                const uint2 v = *reinterpret_cast<const uint2*>(src);
                x[0] = bf16_lo(v.x), x[1] = bf16_hi(v.x), x[2] = bf16_lo(v.y), x[3] = bf16_hi(v.y);
            } else {
#pragma unroll
                for (int i = 0; i < kMaxPer; ++i)
                    if (i < per) x[i] = __uint_as_float((uint32_t)src[i] << 16);
            }
#pragma unroll
            for (int i = 0; i < kMaxPer; ++i)
                if (i < per) amax = fmaxf(amax, fabsf(x[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // fp32 divisions, correctly rounded: for a bf16 amax neither amax / 448 nor 448 / amax lies within
        // 2^-53 (relative) of an fp32 rounding midpoint (448 = 7 * 2^6), so these equal the fp32
        // roundings of the definition's fp64 scale and of its reciprocal
        const float s32 = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        const float r = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
        if (row < nrows) {
            uint8_t* dst = a.codes + row * a.d + lane * per;
            uint8_t c[kMaxPer];
#pragma unroll
            for (int i = 0; i < kMaxPer; ++i)
                if (i < per) c[i] = e4m3_code(x[i], r, amax);
            if (per == 4)
                *reinterpret_cast<uint32_t*>(dst) = c[0] | (c[1] << 8) | (c[2] << 16) | ((uint32_t)c[3] << 24);
            else
                for (int i = 0; i < per; ++i) dst[i] = c[i];
        }
        if (lane == 0) {
            a.scales[(int64_t)h * a.N_pad + n] = s32;
            if (a.rscales) a.rscales[(int64_t)h * a.N_pad + n] = r;
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
