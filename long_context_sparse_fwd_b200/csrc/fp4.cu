// fp4.cu -- bf16 rows to MXFP4, the operand format of the FP4 lightning indexer (axbrief digest
// "Compressed attention and a new optimizer": MXFP4 on the indexer's query-key path; insight.ai.kr
// digest of the HF blog: the indexer stored in FP4).
//
// OCP Microscaling MXFP4: blocks of 32 consecutive channels share an E8M0 scale 2^(e-127); elements are
// E2M1 (0, 0.5, 1, 1.5, 2, 3, 4, 6 and a sign bit). Per block: amax = max |x|; e = 0 when amax = 0,
// else e = clamp(floor(log2 amax) - 2 + 127, 0, 254); each element is x / 2^(e-127) rounded to the
// nearest E2M1 value, ties to the even code, saturating at 6, and a value rounding to zero is stored as
// +0. Two elements per byte, channel 2i in the low nibble.
//
// One thread per block of 32 channels: 64 bytes in, 16 code bytes and one scale byte out.
#include "kernels.cuh"

namespace csa {

namespace {

__device__ __forceinline__ uint32_t e2m1_code(float q)
{
    const float a = fabsf(q);
    // midpoints between consecutive E2M1 values; on a midpoint the even code (upper for even c) wins
    uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
    return m | (q < 0.f && m != 0u ? 8u : 0u);
}

__global__ void __launch_bounds__(256)
quantize_mxfp4_kernel(const uint16_t *__restrict__ x, int64_t nblocks, int nblk, uint8_t *__restrict__ codes,
                      uint8_t *__restrict__ scales)
{
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= nblocks) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + g * 32);
    uint32_t wv[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = src[i];
        wv[4 * i] = v.x;
        wv[4 * i + 1] = v.y;
        wv[4 * i + 2] = v.z;
        wv[4 * i + 3] = v.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf_lo(wv[i])), fabsf(bf_hi(wv[i]))));
    const int e = amax > 0.f ? min(max(ilogbf(amax) - 2 + 127, 0), 254) : 0;
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {   // word i holds channels 2i, 2i+1 -> byte i of the block's codes
        const uint32_t lo = e2m1_code(ldexpf(bf_lo(wv[i]), 127 - e));
        const uint32_t hi = e2m1_code(ldexpf(bf_hi(wv[i]), 127 - e));
        out[i >> 2] |= (lo | (hi << 4)) << (8 * (i & 3));
    }
    reinterpret_cast<uint4 *>(codes)[g] = make_uint4(out[0], out[1], out[2], out[3]);
    scales[g] = (uint8_t)e;
    (void)nblk;
}

}  // namespace

cudaError_t launch_quantize_mxfp4(const uint16_t *x, int64_t rows, int cols, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t stream)
{
    const int64_t nblocks = rows * (cols / 32);
    if (nblocks == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((nblocks + 255) / 256);
    quantize_mxfp4_kernel<<<grid, 256, 0, stream>>>(x, nblocks, cols / 32, codes, scales);
    return cudaGetLastError();
}

}  // namespace csa
