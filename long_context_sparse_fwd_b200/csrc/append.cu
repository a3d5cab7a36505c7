// append.cu -- the compressor's decode step: one new token per sequence enters the pooling state,
// and when it closes a window the pooled entry is written to the entry cache.
//
// What it computes (Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention": CSA
// pools every m tokens over overlapping windows, HCA over non-overlapping windows of m'; section
// "Cache layers": the compressed buffers keep the tokens of the window still open; the insight.ai.kr
// digest of the HF blog: softmax gate with a learned position bias, FP8 entries with BF16 rope dims):
// the token at position P is written into a per-sequence ring of the last L tokens (slot P mod L).
// When (P+1) is a multiple of m, entry w = (P+1)/m - 1 pools positions [(w+1)m - L, (w+1)m) of the
// ring (positions below 0 dropped) exactly as the prefill compressor does, is rotated at w*m with
// theta_cmp, and is stored as bf16, or as E4M3 codes times a per-entry scale (amax/448 over the
// non-rope channels) with the rope channels in bf16. The token's own row rotated at P with theta_tok
// goes to the window ring at slot (W-1-P) mod W: the decode attention treats the window as a set, and
// while fewer than W tokens exist the valid rows are the last ones, as the decode call expects.
//
// One CTA per sequence, one thread per 8 channels (16-byte vectors); the FP8 scale needs the CTA-wide
// maximum of the entry's non-rope channels.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace csa {

namespace {

constexpr int APPEND_THREADS = 64;   // D <= 512: one thread per 8 channels

__global__ void __launch_bounds__(APPEND_THREADS)
compress_append_kernel(AppendArgs a)
{
    __shared__ float red[APPEND_THREADS / 32];
    const int64_t b = blockIdx.x;
    const int chunks = a.D >> 3;
    const int c = threadIdx.x;
    const bool active = c < chunks;
    const int d0 = c << 3;
    const int64_t P = a.P;
    const int slot = (int)(P % a.L);
    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
    if (active) {
        xv = *reinterpret_cast<const uint4 *>(a.x_new + b * a.D + d0);
        const uint4 gv = *reinterpret_cast<const uint4 *>(a.g_new + b * a.D + d0);
        *reinterpret_cast<uint4 *>(a.state_x + (b * a.L + slot) * a.D + d0) = xv;
        *reinterpret_cast<uint4 *>(a.state_g + (b * a.L + slot) * a.D + d0) = gv;
        if (a.win != nullptr) {   // the token's window row, rotated at P with theta_tok
            uint4 v = xv;
            if (d0 >= a.D - a.r) {
                uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int p = (d0 + 2 * e - (a.D - a.r)) >> 1;
                    float cs, sn;
                    rope_cos_sin((double)P, p, a.r, a.log2_theta_tok, &cs, &sn);
                    const float x0 = bf_lo(vw[e]), x1 = bf_hi(vw[e]);
                    vw[e] = pack_bf2(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
                }
                v = make_uint4(vw[0], vw[1], vw[2], vw[3]);
            }
            const int64_t wslot = ((int64_t)a.W - 1 - P % a.W + a.W) % a.W;
            *reinterpret_cast<uint4 *>(a.win + (b * a.W + wslot) * a.D + d0) = v;
        }
    }
    if ((P + 1) % a.m != 0) return;   // no window closes at this position (uniform over the CTA)
    const int64_t w = (P + 1) / a.m - 1;
    if (w >= a.Tcap) return;          // the caller's cache is full: checked on the host
    // pool positions [(w+1)m - L, (w+1)m) = [P + 1 - L, P] from the ring, in position order
    float out[8];
    if (active) {
        float mx[8], l[8], acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; l[e] = 0.f; acc[e] = 0.f; }
        const int64_t start = P + 1 - a.L;
        for (int64_t j = start < 0 ? 0 : start; j <= P; ++j) {
            const int s = (int)(j % a.L);
            const uint4 g = *reinterpret_cast<const uint4 *>(a.state_g + (b * a.L + s) * a.D + d0);
            const uint4 v = *reinterpret_cast<const uint4 *>(a.state_x + (b * a.L + s) * a.D + d0);
            const float bias = a.bias[j - start];
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float z = ((e & 1) ? bf_hi(gw[e >> 1]) : bf_lo(gw[e >> 1])) + bias;
                const float x = (e & 1) ? bf_hi(vw[e >> 1]) : bf_lo(vw[e >> 1]);
                if (z > mx[e]) {
                    const float corr = expf(mx[e] - z);
                    l[e] = l[e] * corr + 1.f;
                    acc[e] = acc[e] * corr + x;
                    mx[e] = z;
                } else {
                    const float p = expf(z - mx[e]);
                    l[e] += p;
                    acc[e] += p * x;
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = acc[e] / l[e];
        if (d0 >= a.D - a.r) {   // rotate at the entry position w*m with theta_cmp
            const double pos = (double)(w * a.m);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const int p = (d0 + e - (a.D - a.r)) >> 1;
                float cs, sn;
                rope_cos_sin(pos, p, a.r, a.log2_theta_cmp, &cs, &sn);
                const float x0 = out[e], x1 = out[e + 1];
                out[e] = x0 * cs - x1 * sn;
                out[e + 1] = x0 * sn + x1 * cs;
            }
        }
    }
    if (a.C != nullptr) {   // bf16 entry
        if (active) {
            uint4 o;
            o.x = pack_bf2(out[0], out[1]);
            o.y = pack_bf2(out[2], out[3]);
            o.z = pack_bf2(out[4], out[5]);
            o.w = pack_bf2(out[6], out[7]);
            *reinterpret_cast<uint4 *>(a.C + (b * a.Tcap + w) * a.D + d0) = o;
        }
        return;
    }
    // FP8 entry: scale = amax / 448 over the non-rope channels, codes rounded to nearest (saturating)
    const bool nope = active && d0 < a.D - a.r;
    float amax = 0.f;
    if (nope) {
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(out[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < APPEND_THREADS / 32; ++i) amax = fmaxf(amax, red[i]);
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    const int64_t row = b * a.Tcap + w;
    if (threadIdx.x == 0) a.c8_scale[row] = scale;
    if (nope) {
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t code = (uint32_t)__nv_cvt_float_to_fp8(out[e] / scale, __NV_SATFINITE, __NV_E4M3);
            if (e < 4) lo |= code << (8 * e);
            else hi |= code << (8 * (e - 4));
        }
        *reinterpret_cast<uint2 *>(a.c8 + row * (a.D - a.r) + d0) = make_uint2(lo, hi);
    } else if (active) {
        uint4 o;
        o.x = pack_bf2(out[0], out[1]);
        o.y = pack_bf2(out[2], out[3]);
        o.z = pack_bf2(out[4], out[5]);
        o.w = pack_bf2(out[6], out[7]);
        *reinterpret_cast<uint4 *>(a.c_rope + row * a.r + (d0 - (a.D - a.r))) = o;
    }
}

}  // namespace

cudaError_t launch_compress_append(const AppendArgs &a, cudaStream_t stream)
{
    if (a.B == 0) return cudaSuccess;
    compress_append_kernel<<<(unsigned)a.B, APPEND_THREADS, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
