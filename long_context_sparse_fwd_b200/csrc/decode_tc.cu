// decode_tc.cu -- decode-step lightning indexer and exact top-k (Hugging Face Transformers docs
// "DeepSeek-V4", section "Hybrid attention", CSA: the indexer scores the query against the
// compressed pool and keeps index_topk entries; the insight.ai.kr digest of the HF blog: ReLU
// multi-head dot product). One new query per sequence sees every one of its T cached entries:
//     I[b,s] = sum_h w[b,h] * ReLU(qI[b,h,:] . kI[b,s,:])
//
// The k^I stream (T x d_I bf16 per sequence: 8 MiB at 128K context, 64 MiB at 1M) dominates the
// step, so the score kernel is built to run at HBM speed: one persistent CTA per SM streams a
// contiguous range of k^I tiles through a 6-deep TMA ring (128-byte swizzle), the tensor cores form
// D[s,h] = kI[s,:] . qI[b,h,:] (entries on TMEM lanes, M=128 x N=HI), and each epilogue thread
// reduces its entry's HI heads in registers and writes one fp32 score.
//
// Top-k is exact and deterministic: the scan also records each sequence's key range; a histogram of
// the leading differing key bits over all of a sequence's scores finds the threshold bin; the
// entries above it are marked in a bitmap and those in it collected and ranked, and the selection
// is written in ascending index order (ties to the smaller index). Up to 32768 entries per sequence
// one CTA does all of it with the sequence's keys in shared memory; past that, chunks of 8192
// entries are histogrammed and collected by many CTAs and one CTA per sequence ranks and writes.
#include <algorithm>
#include <cstring>

#include "kernels.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

constexpr int BM = 128;
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int MAX_STAGES = 6;
constexpr int NACC = 4;                // TMEM accumulators (each HI columns) in flight

struct ScoreParams {
    const float *w;      // [B, HI]
    float *scores;       // [B, T]
    uint32_t *keymax;    // [B] largest order-preserving score key (zero before the scan)
    uint32_t *nkeymin;   // [B] largest complemented key, i.e. ~(smallest key) (zero before the scan)
    int32_t *status;
    uint4 *zero;         // top-k counters, histograms and bitmaps: cleared here for the kernels after
    int64_t zero_n16;    // (16-byte words)
    int64_t T, G;        // entries per sequence; total tiles (B * tiles per sequence)
    int HI, dI, stages, tps;
};

// (sequence, tile within the sequence) of a CTA's consecutive tiles, advanced without a 64-bit division
// per tile (one costs some 450 cycles of a role's per-tile loop).
struct TileCursor {
    int64_t b;
    int it, tps;
    __device__ TileCursor(int64_t g0, int tps_) : b(g0 / tps_), it((int)(g0 - (g0 / tps_) * tps_)), tps(tps_) {}
    __device__ __forceinline__ void next()
    {
        if (++it == tps) {
            it = 0;
            ++b;
        }
    }
};

// Epilogue of the scan (four warps, 128 threads, one TMEM lane quarter each): each thread owns one entry
// of the tile, reduces its HI heads (w-weighted ReLU) in registers and writes one fp32 score; it also
// tracks the sequence's key range for the top-k and clears the chunked top-k's counters.
// NA accumulators in TMEM (tile i in accumulator i % NA); WREG: the index weights of the current sequence
// are held in registers (else read from shared memory, for a kernel that runs two CTAs per SM).
template <int NA, bool WREG>
__device__ __forceinline__ void scan_epilogue(const ScoreParams &p, uint32_t tmem, uint64_t *tfull, uint64_t *tempty,
                                              volatile int *abort, float *sw, int64_t g_lo, int ntiles, int warp,
                                              int lane, int etid)
{
    const int quarter = warp & 3;
    const uint32_t taddr0 = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int64_t i = (int64_t)blockIdx.x * EPI_THREADS + etid; i < p.zero_n16; i += (int64_t)gridDim.x * EPI_THREADS)
        p.zero[i] = make_uint4(0u, 0u, 0u, 0u);
    float wr[WREG ? 64 : 1];   // index weights of the current sequence (HI == 64 keeps them in registers)
    // range of the score keys of the current sequence seen by this thread, merged into the
    // sequence's global range (for the top-k's histogram) whenever the sequence changes
    uint32_t kmax = 0u, knmin = 0u;
    int64_t b_cur = -1;
    auto flush_range = [&]() {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
            knmin = max(knmin, __shfl_xor_sync(0xffffffffu, knmin, o));
        }
        if (lane == 0 && b_cur >= 0) {
            atomicMax(p.keymax + b_cur, kmax);
            atomicMax(p.nkeymin + b_cur, knmin);
        }
        kmax = 0u;
        knmin = 0u;
    };
    TileCursor cur(g_lo, p.tps);
    for (int i = 0; i < ntiles; ++i, cur.next()) {
        const int64_t b = cur.b;
        const int it = cur.it;
        if (b != b_cur) {
            flush_range();
            b_cur = b;
        }
        if (i == 0 || it == 0) {   // index weights of the new sequence
            named_barrier_sync(1, EPI_THREADS);
            for (int h = etid; h < p.HI; h += EPI_THREADS) sw[h] = p.w[b * p.HI + h];
            named_barrier_sync(1, EPI_THREADS);
            if (WREG && p.HI == 64) {
#pragma unroll
                for (int h = 0; h < (WREG ? 64 : 1); ++h) wr[h] = sw[h];
            }
        }
        const int buf = i % NA;
        if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (i / NA) & 1, abort, p.status))) break;
        tc_fence_after();
        float acc = 0.f;
        if (p.HI == 64) {
            float v0[32], v1[32];
            tmem_ld32(taddr0 + buf * 64, v0);        // both loads in flight, one wait
            tmem_ld32(taddr0 + buf * 64 + 32, v1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&tempty[buf]);               // the accumulator may be reused from here
            float a1 = 0.f, a2 = 0.f, a3 = 0.f;   // four independent chains: the sum is latency-bound otherwise
            if constexpr (WREG) {
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    acc = fmaf(wr[jj], fmaxf(v0[jj], 0.f), acc);
                    a1 = fmaf(wr[jj + 1], fmaxf(v0[jj + 1], 0.f), a1);
                    a2 = fmaf(wr[32 + jj], fmaxf(v1[jj], 0.f), a2);
                    a3 = fmaf(wr[33 + jj], fmaxf(v1[jj + 1], 0.f), a3);
                }
            } else {
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    const float2 w0 = *reinterpret_cast<const float2 *>(sw + jj);
                    const float2 w1 = *reinterpret_cast<const float2 *>(sw + 32 + jj);
                    acc = fmaf(w0.x, fmaxf(v0[jj], 0.f), acc);
                    a1 = fmaf(w0.y, fmaxf(v0[jj + 1], 0.f), a1);
                    a2 = fmaf(w1.x, fmaxf(v1[jj], 0.f), a2);
                    a3 = fmaf(w1.y, fmaxf(v1[jj + 1], 0.f), a3);
                }
            }
            acc = (acc + a1) + (a2 + a3);
        } else {
            for (int h0 = 0; h0 < p.HI; h0 += 16) {
                if (h0 + 32 <= p.HI) {
                    float v[32];
                    tmem_ld32(taddr0 + buf * p.HI + h0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) acc = fmaf(sw[h0 + jj], fmaxf(v[jj], 0.f), acc);
                    h0 += 16;
                } else {
                    float v[16];
                    tmem_ld16(taddr0 + buf * p.HI + h0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) acc = fmaf(sw[h0 + jj], fmaxf(v[jj], 0.f), acc);
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
        }
        const int64_t s = (int64_t)it * BM + quarter * 32 + lane;
        if (s < p.T) {
            p.scores[b * p.T + s] = acc + 0.0f;
            const uint32_t key = score_key(acc);
            kmax = max(kmax, key);
            knmin = max(knmin, ~key);
        }
    }
    flush_range();
}

// Persistent: CTA c takes the contiguous tile range [c*G/n, (c+1)*G/n) of the flat list
// (sequence-major, 128 entries per tile), so the HBM stream never idles on a wave tail. q^I of the
// current sequence is double-buffered; a range crosses at most a few sequence boundaries.
__global__ void __launch_bounds__(NUM_THREADS, 2)
decode_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        ScoreParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int kchunks = p.dI / 64;
    const uint32_t b_bytes = (uint32_t)kchunks * p.HI * 128;
    const uint32_t a_bytes = (uint32_t)kchunks * BM * 128;
    uint8_t *sB = smem;                                   // [2][b_bytes]
    uint8_t *sA = sB + 2 * b_bytes;
    float *sw = reinterpret_cast<float *>(sA + (size_t)p.stages * a_bytes);   // [HI] of the current sequence
    uint64_t *bars = reinterpret_cast<uint64_t *>(sw + 256);
    uint64_t *full = bars, *empty = bars + 8, *tfull = bars + 16, *tempty = bars + 20;   // tfull/tempty: [NACC]
    uint64_t *qfull = bars + 24, *qempty = bars + 26;     // [2] each
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 28);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 29);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g_lo = (int64_t)blockIdx.x * p.G / gridDim.x;
    const int64_t g_hi = (int64_t)(blockIdx.x + 1) * p.G / gridDim.x;
    const int ntiles = (int)(g_hi - g_lo);
    const int64_t b_first = g_lo / p.tps;
    const uint32_t tcols = p.HI * NACC <= 32 ? 32 : (p.HI * NACC <= 64 ? 64 : (p.HI * NACC <= 128 ? 128 : (p.HI * NACC <= 256 ? 256 : 512)));

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
        }
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    grid_launch_dependents();   // the top-k kernels may be scheduled as this grid's CTAs finish

    if (warp == 0) {
        if (ntiles > 0) {
            const uint64_t pol_stream = policy_evict_first();   // k^I is read once per step
            int issued = 0, nseg = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, j = (int)(b - b_first);
                if (i == 0 || it == 0) {   // a new sequence: its q^I into buffer j & 1
                    if (!__all_sync(0xffffffffu, mbar_wait(&qempty[j & 1], ((j >> 1) & 1) ^ 1, abort, p.status))) break;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&qfull[j & 1], b_bytes);
                        for (int c = 0; c < kchunks; ++c)
                            tma_load_2d(sB + (j & 1) * b_bytes + c * p.HI * 128, &tm_q, &qfull[j & 1], c * 64,
                                        (int)(b * p.HI));
                    }
                    __syncwarp();
                    nseg = j + 1;
                }
                const int st = i % p.stages;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((i / p.stages) & 1) ^ 1, abort, p.status))) break;
                const int y = (int)(b * p.T + (int64_t)it * BM);
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[st], a_bytes);
                    for (int c = 0; c < kchunks; ++c)
                        tma_load_2d_hint(sA + st * a_bytes + c * BM * 128, &tm_k, &full[st], c * 64, y, pol_stream);
                }
                __syncwarp();
                issued = i + 1;
            }
            // never leave with copies in flight into this CTA's shared memory
            for (int j = max(0, nseg - 2); j < nseg; ++j)
                mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status, 100000000ull);
            for (int i = max(0, issued - p.stages); i < issued; ++i)
                mbar_wait(&full[i % p.stages], (i / p.stages) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp == 1) {
        if (ntiles > 0) {
            const uint32_t idesc = idesc_bf16(BM, p.HI);
            const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
            int issued = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, j = (int)(b - b_first);
                if (i == 0 || it == 0)
                    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status))) break;
                const int st = i % p.stages, buf = i % NACC;
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((i / NACC) & 1) ^ 1, abort, p.status))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (i / p.stages) & 1, abort, p.status))) break;
                tc_fence_after();
                const uint64_t dBj = dB + (((j & 1) * b_bytes) >> 4);
                if (elect_one()) {   // one lane issues; the loop itself runs warp-wide (uniform operands)
                    for (int c = 0; c < kchunks; ++c)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + buf * p.HI, dA + ((st * a_bytes + c * BM * 128 + ks * 32) >> 4),
                                     dBj + ((c * p.HI * 128 + ks * 32) >> 4), idesc, (c | ks) != 0);
                    mma_commit(&empty[st]);
                    mma_commit(&tfull[buf]);
                    if (i + 1 == ntiles || it + 1 == p.tps) mma_commit(&qempty[j & 1]);   // done with this q^I
                }
                __syncwarp();
                issued = i + 1;
            }
            if (issued > 0)
                mbar_wait(&tfull[(issued - 1) % NACC], ((issued - 1) / NACC) & 1, abort, p.status, 100000000ull);
        }
    } else {
        scan_epilogue<NACC, false>(p, tmem, tfull, tempty, abort, sw, g_lo, ntiles, warp, lane, threadIdx.x - 64);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

// ---- the same scan on MXFP4 operands ------------------------------------------------------------------
//
// q^I and k^I arrive as MXFP4 (E2M1 codes, two per byte, and one E8M0 scale per 32 channels). A
// producer warp brings each 128-entry tile of k^I codes (dI/2 bytes per entry) into a ring of staging
// buffers by TMA; four converter warps (one entry row per thread) dequantise it into the bf16
// 128-byte-swizzled A tile the MMA reads, and at each new sequence dequantise its q^I into the B
// operand. Every E2M1 value times a power of two is exact in bf16, so the bf16 MMA with fp32
// accumulation computes the scores of the dequantised operands. The epilogue is the bf16 scan's.

constexpr int F4_THREADS = 320;        // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue, warps 6-9 convert
constexpr int F4_CONV0 = 6;
constexpr int F4_CST = 6;              // code staging buffers

struct Fp4Params {
    ScoreParams sp;
    const uint8_t *qc, *qs;            // q^I codes [B, HI, dI/2], scales [B, HI, dI/32]
    const uint8_t *ks;                 // k^I scales [B*T, dI/32]
    int64_t rows;                      // B*T
};

// The two dequantised values of a code byte (channel 2i in the low half) as a bf16 pair, unscaled.
__device__ __forceinline__ uint32_t e2m1_pair_bits(uint32_t byte)
{
    auto one = [](uint32_t n) -> uint32_t {
        const uint32_t m = n & 7u;
        uint32_t f;   // fp32 bits of the magnitude
        if (m == 0u) f = 0u;
        else if (m == 1u) f = 126u << 23;                                   // 0.5
        else f = (((m >> 1) + 126u) << 23) | ((m & 1u) << 22);              // (1 + mant/2) 2^(exp-1)
        f |= (n & 8u) && m != 0u ? 0x80000000u : 0u;
        return f >> 16;                                                     // exact: bf16 keeps the top half
    };
    return one(byte & 15u) | (one(byte >> 4) << 16);
}

// 2^(e-127) as a bf16 pair (exact for every E8M0 value below 255; e = 0 is the subnormal 2^-127)
__device__ __forceinline__ __nv_bfloat162 e8m0_scale2(uint32_t e)
{
    const uint32_t f = e != 0u ? (e << 23) : 0x00400000u;
    const uint32_t h2 = (f >> 16) | (f & 0xffff0000u);
    __nv_bfloat162 r;
    memcpy(&r, &h2, 4);
    return r;
}

__global__ void __launch_bounds__(F4_THREADS, 1)
decode_scores_fp4_kernel(const __grid_constant__ CUtensorMap tm_kc, Fp4Params f)
{
    const ScoreParams &p = f.sp;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int kchunks = p.dI / 64;
    const uint32_t a_bytes = (uint32_t)kchunks * BM * 128;   // bf16 A tile
    const uint32_t b_bytes = (uint32_t)kchunks * p.HI * 128; // bf16 q^I
    const uint32_t c_row = (uint32_t)p.dI / 2;               // code bytes per entry
    const uint32_t c_bytes = c_row * BM;
    uint8_t *sA = smem;                                      // [2][a_bytes]
    uint8_t *sB = sA + 2 * a_bytes;                          // [2][b_bytes]
    uint8_t *sC = sB + 2 * b_bytes;                          // [F4_CST][c_bytes]
    float *sw = reinterpret_cast<float *>(sC + F4_CST * c_bytes);   // [256]
    uint32_t *lut = reinterpret_cast<uint32_t *>(sw + 256);         // [256] code byte -> bf16 pair
    uint64_t *bars = reinterpret_cast<uint64_t *>(lut + 256);
    uint64_t *cfull = bars, *cempty = bars + 8;              // [F4_CST]
    uint64_t *afull = bars + 16, *aempty = bars + 18;        // [2]
    uint64_t *qfull = bars + 20, *qempty = bars + 22;        // [2]
    uint64_t *tfull = bars + 24, *tempty = bars + 28;        // [NACC]
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 32);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 33);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g_lo = (int64_t)blockIdx.x * p.G / gridDim.x;
    const int64_t g_hi = (int64_t)(blockIdx.x + 1) * p.G / gridDim.x;
    const int ntiles = (int)(g_hi - g_lo);
    const int64_t b_first = g_lo / p.tps;
    const uint32_t tcols = p.HI * NACC <= 32 ? 32 : (p.HI * NACC <= 64 ? 64 : (p.HI * NACC <= 128 ? 128 : (p.HI * NACC <= 256 ? 256 : 512)));
    const int ctid = threadIdx.x - F4_CONV0 * 32;            // converter thread: entry row of the tile

    if (threadIdx.x == 0) {
        for (int i = 0; i < F4_CST; ++i) { mbar_init(&cfull[i], 1); mbar_init(&cempty[i], 128); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&afull[i], 128);
            mbar_init(&aempty[i], 1);
            mbar_init(&qfull[i], 128);
            mbar_init(&qempty[i], 1);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
        }
        *abort = 0;
        fence_barrier_init();
    }
    if (ctid >= 0) {
        lut[ctid] = e2m1_pair_bits((uint32_t)ctid);
        lut[ctid + 128] = e2m1_pair_bits((uint32_t)ctid + 128u);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    grid_launch_dependents();   // the top-k may be scheduled as this grid's CTAs finish

    if (warp == 0) {
        // ---------------- TMA producer: k^I code tiles ----------------
        if (ntiles > 0) {
            if (elect_one()) prefetch_tmap(&tm_kc);
            __syncwarp();
            const uint64_t pol_stream = policy_evict_first();
            int issued = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, st = i % F4_CST;
                if (!__all_sync(0xffffffffu, mbar_wait(&cempty[st], ((i / F4_CST) & 1) ^ 1, abort, p.status))) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&cfull[st], c_bytes);
                    tma_load_2d_hint(sC + st * c_bytes, &tm_kc, &cfull[st], 0, (int)(b * p.T + (int64_t)it * BM), pol_stream);
                }
                __syncwarp();
                issued = i + 1;
            }
            for (int i = max(0, issued - F4_CST); i < issued; ++i)   // no copy in flight at exit
                mbar_wait(&cfull[i % F4_CST], (i / F4_CST) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (ntiles > 0) {
            const uint32_t idesc = idesc_bf16(BM, p.HI);
            const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
            int issued = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, j = (int)(b - b_first);
                if (i == 0 || it == 0)
                    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status))) break;
                const int buf = i % NACC, ab = i & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((i / NACC) & 1) ^ 1, abort, p.status))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(&afull[ab], (i >> 1) & 1, abort, p.status))) break;
                tc_fence_after();
                const uint64_t dBj = dB + (((j & 1) * b_bytes) >> 4);
                if (elect_one()) {
                    for (int c = 0; c < kchunks; ++c)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + buf * p.HI, dA + ((ab * a_bytes + c * BM * 128 + ks * 32) >> 4),
                                     dBj + ((c * p.HI * 128 + ks * 32) >> 4), idesc, (c | ks) != 0);
                    mma_commit(&aempty[ab]);
                    mma_commit(&tfull[buf]);
                    if (i + 1 == ntiles || it + 1 == p.tps) mma_commit(&qempty[j & 1]);
                }
                __syncwarp();
                issued = i + 1;
            }
            if (issued > 0)
                mbar_wait(&tfull[(issued - 1) % NACC], ((issued - 1) / NACC) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp < F4_CONV0) {
        scan_epilogue<NACC, true>(p, tmem, tfull, tempty, abort, sw, g_lo, ntiles, warp, lane, threadIdx.x - 64);
    } else {
        // ---------------- converters: thread ctid dequantises entry row ctid of each tile ----------------
        const int nblk = p.dI / 32;                           // scale blocks per row
        TileCursor cur(g_lo, p.tps);
        for (int i = 0; i < ntiles; ++i, cur.next()) {
            const int64_t b = cur.b;
            const int it = cur.it, j = (int)(b - b_first);
            if (i == 0 || it == 0) {
                // q^I of the new sequence into B operand buffer j & 1 (HI rows x dI), once the MMAs
                // of the sequence two back are done with it
                if (!__all_sync(0xffffffffu, mbar_wait(&qempty[j & 1], ((j >> 1) & 1) ^ 1, abort, p.status))) break;
                uint8_t *dst = sB + (j & 1) * b_bytes;
                for (int q = ctid; q < p.HI * nblk; q += 128) {   // one 32-channel block each
                    const int h = q / nblk, blk = q % nblk;
                    const int64_t rq = b * p.HI + h;
                    const uint4 cv = *reinterpret_cast<const uint4 *>(f.qc + rq * (p.dI / 2) + blk * 16);
                    const __nv_bfloat162 sc2 = e8m0_scale2(f.qs[rq * nblk + blk]);
                    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {   // 8 channels per 16-byte unit
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t pr = lut[(cw[u] >> (8 * e)) & 255u];
                            const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&pr), sc2);
                            o[e] = *reinterpret_cast<const uint32_t *>(&v);
                        }
                        const int ch = blk * 32 + u * 8, c = ch >> 6, uu = (ch & 63) >> 3;
                        *reinterpret_cast<uint4 *>(dst + c * p.HI * 128 + h * 128 + ((uu ^ (h & 7)) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                fence_async_smem();
                mbar_arrive(&qfull[j & 1]);
            }
            const int st = i % F4_CST, ab = i & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&cfull[st], (i / F4_CST) & 1, abort, p.status))) break;
            // Thread ctid takes 32-channel block u = ctid % nblk of rows ctid / nblk + k * (128 / nblk),
            // k < nblk: a warp reads 512 contiguous staging bytes per pass.
            const int rpp = 128 / nblk, u = ctid % nblk;
            uint4 cv[4];
            uint32_t sb[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (k >= nblk) break;
                const int r = k * rpp + ctid / nblk;
                cv[k] = *reinterpret_cast<const uint4 *>(sC + st * c_bytes + r * c_row + u * 16);
                const int64_t grow = b * p.T + (int64_t)it * BM + r;
                sb[k] = grow < f.rows ? (uint32_t)f.ks[grow * nblk + u] : 0u;
            }
            mbar_arrive(&cempty[st]);   // the staging buffer may be refilled
            if (!__all_sync(0xffffffffu, mbar_wait(&aempty[ab], ((i >> 1) & 1) ^ 1, abort, p.status))) break;
            uint8_t *dst = sA + ab * a_bytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (k >= nblk) break;
                const int r = k * rpp + ctid / nblk;
                const __nv_bfloat162 sc2 = e8m0_scale2(sb[k]);
                const uint32_t cw[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {   // channels 32u + 8q .. +7: bytes 4q .. 4q+3 of the block
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t pr = lut[(cw[q] >> (8 * e)) & 255u];
                        const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&pr), sc2);
                        o[e] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    const int ch = u * 32 + q * 8, c = ch >> 6, uu = (ch & 63) >> 3;
                    *reinterpret_cast<uint4 *>(dst + c * BM * 128 + r * 128 + ((uu ^ (r & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            fence_async_smem();   // generic-proxy writes, read by the MMA through the async proxy
            mbar_arrive(&afull[ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

// ---- the MXFP4 scan on the block-scaled tensor-core MMA ---------------------------------------------
//
// The same scan with the MXFP4 operands fed to tcgen05.mma kind::mxf4 directly: packed E2M1 codes in
// shared memory (64-byte rows, 64-byte swizzle, K = 64 channels per instruction) and one E8M0 scale per
// 32 channels in TMEM, so nothing is converted and the k^I stream is 68 bytes per entry (64 code bytes,
// 4 scale bytes). In TMEM the scales of matrix row 32 j + r (r < 32) sit in lane r of every lane
// quarter, column j, one byte per 32-channel block: tcgen05.cp replicates a [32 x 16 bytes] matrix whose
// row r holds the scale words of entries r, r + 32, r + 64, r + 96 into the four quarters.
// A tile's codes (128 entries x 64 bytes) and scales (4 bytes per entry) are brought by two loader warps
// with 16- and 4-byte cp.async copies written straight into the MMA's layout: code row t's four 16-byte
// units at u ^ ((t >> 1) & 3) (the 64-byte swizzle), scale word of entry r + 32 j at row r, column j.
// The roles hand each tile over through mbarriers, and with one CTA per SM every role advanced at the pace
// of those handovers rather than of the stream: two CTAs run on each SM, each a pipeline of its own. The q^I
// scales of a sequence (row = head) are gathered by the producer warp into the same arrangement (lane r,
// column j: head r + 32 j). dI = 128 (two instructions per tile), HI <= 64 (N <= 64), T a multiple of 4.

// Two CTAs per SM (two independent tile pipelines): 256 threads and at most 128 registers each, about 96 KB
// of shared memory and 256 TMEM columns per CTA.
constexpr int X4_THREADS = 256;        // warp 0 q^I and its scales, warp 1 MMA and scale copies, warps 2-5
                                       // epilogue, warps 6-7 k^I loads (two code rows per thread)
constexpr int X4_LOADERS = 64;
constexpr int X4_INFLIGHT = 7;         // tiles of copies in flight per loader thread (<= X4_STAGES)
constexpr int X4_STAGES = 10;
constexpr int X4_NACC = 3;             // TMEM accumulators (64 columns each)
constexpr uint32_t X4_A_BYTES = BM * 64;          // 128 entries x 64 code bytes
constexpr uint32_t X4_SF_BYTES = 512;             // [32 x 16 bytes] of scales
constexpr uint32_t X4_SFA_COL = 192, X4_SFB_COL = 208;   // TMEM columns of the scale slots (4 each)
constexpr uint32_t X4_TMEM_COLS = 256;

struct Mxf4Params {
    ScoreParams sp;
    const uint8_t *qs;                 // q^I scales [B, HI, 4]
    const uint8_t *kc;                 // k^I codes [B*T, 64], 16-byte aligned
    const uint8_t *ks;                 // k^I scales [B*T, 4], 16-byte aligned
};

// Asynchronous global -> shared copies through the load path (cp.async), grouped per commit.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint64_t policy)
{
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(policy) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(X4_THREADS, 2)
decode_scores_mxf4_kernel(const __grid_constant__ CUtensorMap tm_qc, Mxf4Params f)
{
    const ScoreParams &p = f.sp;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t b_bytes = (uint32_t)p.HI * 64;
    uint8_t *sA = smem;                                           // [X4_STAGES][X4_A_BYTES]
    uint8_t *sB = sA + X4_STAGES * X4_A_BYTES;                    // [2][4 KB]
    uint8_t *sSFA = sB + 2 * 4096;                                // [X4_STAGES][X4_SF_BYTES]
    uint8_t *sSFB = sSFA + X4_STAGES * X4_SF_BYTES;               // [2][X4_SF_BYTES]
    float *sw = reinterpret_cast<float *>(sSFB + 2 * X4_SF_BYTES);   // [256]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sw + 256);
    uint64_t *full = bars, *empty = bars + X4_STAGES;             // [X4_STAGES]
    uint64_t *tfull = bars + 2 * X4_STAGES, *tempty = tfull + X4_NACC;   // [X4_NACC]
    uint64_t *qfull = tempty + X4_NACC, *qempty = qfull + 2;      // [2]
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(qempty + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(qempty + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g_lo = (int64_t)blockIdx.x * p.G / gridDim.x;
    const int64_t g_hi = (int64_t)(blockIdx.x + 1) * p.G / gridDim.x;
    const int ntiles = (int)(g_hi - g_lo);
    const int64_t b_first = g_lo / p.tps;
    constexpr uint32_t tcols = X4_TMEM_COLS;   // accumulators X4_NACC x HI (HI <= 64) and the scale slots

    if (threadIdx.x == 0) {
        for (int i = 0; i < X4_STAGES; ++i) {
            mbar_init(&full[i], X4_LOADERS);   // every loader thread, once its copies of the tile have landed
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < X4_NACC; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 2);   // the q^I code load (with its bytes) and the gathered scales
            mbar_init(&qempty[i], 1);
        }
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    grid_launch_dependents();   // the top-k may be scheduled as this grid's CTAs finish

    if (warp == 0) {
        // ---------------- q^I and its scales, per sequence ----------------
        if (ntiles > 0) {
            if (elect_one()) prefetch_tmap(&tm_qc);
            __syncwarp();
            int nseg = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, j = (int)(b - b_first);
                if (i == 0 || it == 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&qempty[j & 1], ((j >> 1) & 1) ^ 1, abort, p.status))) break;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&qfull[j & 1], b_bytes);
                        tma_load_2d(sB + (j & 1) * 4096, &tm_qc, &qfull[j & 1], 0, (int)(b * p.HI));
                    }
                    // scales of q^I: lane r writes row r = the 4-byte scale words of heads r + 32 c
                    uint32_t wq[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int h = lane + 32 * c;
                        wq[c] = h < p.HI ? *reinterpret_cast<const uint32_t *>(f.qs + (b * p.HI + h) * 4) : 0u;
                    }
                    *reinterpret_cast<uint4 *>(sSFB + (j & 1) * X4_SF_BYTES + lane * 16) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&qfull[j & 1]);
                    nseg = j + 1;
                }
            }
            // never leave with copies in flight into this CTA's shared memory
            for (int j = max(0, nseg - 2); j < nseg; ++j)
                mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: scale copies into TMEM, then two block-scaled MMAs per tile ----------
        if (ntiles > 0) {
            const uint32_t id0 = idesc_mxf4(BM, p.HI, 0), id2 = idesc_mxf4(BM, p.HI, 2);
            const uint64_t dA = sdesc_sw64(smem_u32(sA), 512), dB = sdesc_sw64(smem_u32(sB), 512);
            int issued = 0;
            TileCursor cur(g_lo, p.tps);
            for (int i = 0; i < ntiles; ++i, cur.next()) {
                const int64_t b = cur.b;
                const int it = cur.it, j = (int)(b - b_first);
                const uint32_t sfb = tmem + X4_SFB_COL + (uint32_t)(j & 1) * 4;
                if (i == 0 || it == 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status))) break;
                    tc_fence_after();
                    if (elect_one()) tmem_cp_32x128b_x4(sfb, sdesc_plain(smem_u32(sSFB + (j & 1) * X4_SF_BYTES), 16, 128));
                    __syncwarp();
                }
                const int st = i % X4_STAGES, buf = i % X4_NACC;
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((i / X4_NACC) & 1) ^ 1, abort, p.status))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (i / X4_STAGES) & 1, abort, p.status))) break;
                tc_fence_after();
                const uint32_t sfa = tmem + X4_SFA_COL + (uint32_t)buf * 4;
                if (elect_one()) {
                    tmem_cp_32x128b_x4(sfa, sdesc_plain(smem_u32(sSFA + st * X4_SF_BYTES), 16, 128));
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)   // channels 64 ks .. 64 ks + 63: scale bytes 2 ks, 2 ks + 1
                        mma_mxf4(tmem + buf * p.HI, dA + ((st * X4_A_BYTES + ks * 32) >> 4),
                                 dB + (((j & 1) * 4096 + ks * 32) >> 4), ks ? id2 : id0,
                                 sfa | ((uint32_t)(2 * ks) << 30), sfb | ((uint32_t)(2 * ks) << 30), ks != 0);
                    mma_commit(&empty[st]);
                    mma_commit(&tfull[buf]);
                    if (i + 1 == ntiles || it + 1 == p.tps) mma_commit(&qempty[j & 1]);   // done with this q^I
                }
                __syncwarp();
                issued = i + 1;
            }
            if (issued > 0)
                mbar_wait(&tfull[(issued - 1) % X4_NACC], ((issued - 1) / X4_NACC) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp < 6) {
        scan_epilogue<X4_NACC, false>(p, tmem, tfull, tempty, abort, sw, g_lo, ntiles, warp, lane, threadIdx.x - 64);
    } else {
        // ---------------- loads: each thread two code rows of every tile, straight into the swizzled layout ---
        // Row r's four 16-byte units land at u ^ ((r >> 1) & 3) (the 64-byte swizzle); warp 6 also brings
        // the scale words, entry r + 32 j to row r, column j. A thread keeps X4_INFLIGHT tiles of its copies in
        // flight: once the copies of tile i - X4_INFLIGHT + 1 have landed it makes them visible to the tensor
        // core (proxy fence) and arrives on that tile's barrier. Only the tile's own rows are read (T % 4 == 0),
        // rows past the sequence's end keep older contents and their scores are not stored.
        const int t = threadIdx.x - 192;                      // code rows t and t + 64 (= entries of the tile)
        const uint64_t pol_stream = policy_evict_first();    // k^I is read once per step
        int issued = 0;
        TileCursor cur(g_lo, p.tps);
        for (int i = 0; i < ntiles; ++i, cur.next()) {
            const int st = i % X4_STAGES;
            const int64_t b = cur.b;
            const int it = cur.it;
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((i / X4_STAGES) & 1) ^ 1, abort, p.status))) break;
            const int64_t e0 = b * p.T + (int64_t)it * BM;    // first entry of the tile
            const int64_t left = p.T - (int64_t)it * BM;
            const int rows = (int)(left < BM ? left : BM);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = t + rr * X4_LOADERS, rot = (r >> 1) & 3;
                if (r < rows) {
                    const uint8_t *src = f.kc + (e0 + r) * 64;
                    const uint32_t dst = smem_u32(sA + st * X4_A_BYTES + r * 64);
#pragma unroll
                    for (int u = 0; u < 4; ++u) cp_async16(dst + (uint32_t)((u ^ rot) << 4), src + u * 16, pol_stream);
                }
            }
            if (warp == 6) {
                const uint32_t dst = smem_u32(sSFA + st * X4_SF_BYTES + lane * 16);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (lane + 32 * jj < rows) cp_async4(dst + 4 * jj, f.ks + (e0 + lane + 32 * jj) * 4);
            }
            cp_async_commit();
            issued = i + 1;
            if (i >= X4_INFLIGHT - 1) {
                cp_async_wait<X4_INFLIGHT - 1>();
                fence_async_smem();   // generic-proxy writes, read next by tcgen05.cp / tcgen05.mma
                mbar_arrive(&full[(i - X4_INFLIGHT + 1) % X4_STAGES]);
            }
        }
        cp_async_wait<0>();   // never leave with copies in flight into this CTA's shared memory
        fence_async_smem();
        for (int i = max(0, issued - (X4_INFLIGHT - 1)); i < issued; ++i) mbar_arrive(&full[i % X4_STAGES]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

// ---- exact top-k by a histogram of the leading differing key bits ----------------------------------
//
// Keys are the order-preserving uint32 images of the scores. Over a sequence the keys share every bit
// above `top` (the highest bit where its smallest and largest key differ); the histogram digit is the
// (up to) 11 bits [shift, top] below them, so a larger digit means a larger key. The threshold digit
// d* is the largest one whose suffix count reaches k: every key with a larger digit is selected
// outright (a bitmap bit per entry), the keys with digit d* are collected as candidates, and the
// final kernel ranks the candidates (key descending, then entry index ascending) to take the rest.
// Indices come out ascending from the bitmap; ties go to the smaller index.

constexpr int HBINS = 2048;
constexpr int TK_CHUNK = 8192;         // entries per histogram / collect CTA
constexpr int TK_THREADS = 512;
constexpr int FIN_THREADS = 1024;
constexpr int CAND_CAP = 2048;         // candidates ranked directly; more take the exact fallback
constexpr int TK_PER = TK_CHUNK / TK_THREADS;   // scores per thread: all loaded before any is used

struct KeyRange {
    uint32_t prefix_hi;   // the common high bits (bits above top), as in every key
    int shift;            // digit = (key >> shift) & dmask
    uint32_t dmask;
};

__device__ __forceinline__ KeyRange key_range(uint32_t kmax, uint32_t knmin)
{
    const uint32_t lo = ~knmin, hi = kmax;
    KeyRange r;
    const uint32_t diff = lo ^ hi;
    if (diff == 0u) {   // one key value: a single bin
        r.shift = 0;
        r.dmask = 0u;
        r.prefix_hi = hi;
        return r;
    }
    const int top = 31 - __clz(diff);
    r.shift = max(0, top - 10);
    r.dmask = (2u << (top - r.shift)) - 1u;
    r.prefix_hi = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
    return r;
}

__device__ __forceinline__ uint32_t key_digit(uint32_t key, const KeyRange &r) { return (key >> r.shift) & r.dmask; }

// Threshold digit of a sequence from its histogram (block of `nthreads` >= HBINS / 4 threads; every
// thread gets the result): d* and the number of keys with a larger digit. Needs T > k.
__device__ void find_threshold(const uint32_t *hist_g, int k, uint32_t *sh_hist, uint32_t *sh_sums, int *dstar,
                               uint32_t *above)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int i = tid; i < HBINS; i += nt) sh_hist[i] = hist_g[i];
    __syncthreads();
    // thread t < 512 owns bins [4t, 4t+4); suffix sums over the owners from the top
    uint32_t own = 0;
    if (tid < HBINS / 4)
        own = sh_hist[4 * tid] + sh_hist[4 * tid + 1] + sh_hist[4 * tid + 2] + sh_hist[4 * tid + 3];
    if (tid < HBINS / 4) sh_sums[tid] = own;
    __syncthreads();
    if (tid < 32) {   // warp 0: suffix scan of the 512 owner sums (16 per lane)
        uint32_t v[16], tot = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) { v[j] = sh_sums[tid * 16 + j]; tot += v[j]; }
        uint32_t after = tot;   // sums held by higher lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_down_sync(0xffffffffu, after, o);
            if (tid + o < 32) after += x;
        }
        after -= tot;
        uint32_t run = after;
#pragma unroll
        for (int j = 15; j >= 0; --j) {   // exclusive suffix: keys in owners above owner 16*lane+j
            const uint32_t vj = v[j];
            sh_sums[tid * 16 + j] = run;
            run += vj;
        }
    }
    __syncthreads();
    if (tid < HBINS / 4) {
        uint32_t run = sh_sums[tid];   // keys in bins >= 4*tid + 4
        for (int j = 3; j >= 0; --j) {
            const uint32_t c = sh_hist[4 * tid + j];
            if (run < (uint32_t)k && run + c >= (uint32_t)k) {
                sh_sums[HBINS / 4] = (uint32_t)(4 * tid + j);
                sh_sums[HBINS / 4 + 1] = run;
            }
            run += c;
        }
    }
    __syncthreads();
    *dstar = (int)sh_sums[HBINS / 4];
    *above = sh_sums[HBINS / 4 + 1];
    __syncthreads();
}

// Histogram of the digits of one chunk of one sequence's scores, added into the sequence's histogram.
__global__ void __launch_bounds__(TK_THREADS)
topk_hist_kernel(const float *__restrict__ scores, int64_t T, const uint32_t *__restrict__ keymax,
                 const uint32_t *__restrict__ nkeymin, uint32_t *__restrict__ hist)
{
    __shared__ uint32_t sh[HBINS];
    const int b = blockIdx.y;
    for (int i = threadIdx.x; i < HBINS; i += TK_THREADS) sh[i] = 0;
    grid_dependency_wait();   // the scores and key ranges of the scan
    grid_launch_dependents();
    const KeyRange r = key_range(keymax[b], nkeymin[b]);
    __syncthreads();
    const int64_t s0 = (int64_t)blockIdx.x * TK_CHUNK;
    const int n = (int)min((int64_t)TK_CHUNK, T - s0);
    const float *sc = scores + b * T + s0;
    float v[TK_PER];
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        const int i = j * TK_THREADS + threadIdx.x;
        v[j] = i < n ? sc[i] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < TK_PER; ++j)
        if (j * TK_THREADS + (int)threadIdx.x < n) atomicAdd(&sh[key_digit(score_key(v[j]), r)], 1u);
    __syncthreads();
    uint32_t *hg = hist + (int64_t)b * HBINS;
    for (int i = threadIdx.x; i < HBINS; i += TK_THREADS)
        if (sh[i] != 0u) atomicAdd(hg + i, sh[i]);
}

// Entries with a digit above d* set their bitmap bit (one ballot word per warp and 32 entries);
// entries with digit d* are appended to the sequence's candidate list.
__global__ void __launch_bounds__(TK_THREADS)
topk_collect_kernel(const float *__restrict__ scores, int64_t T, int k, const uint32_t *__restrict__ keymax,
                    const uint32_t *__restrict__ nkeymin, const uint32_t *__restrict__ hist, uint32_t *__restrict__ bitmap,
                    uint32_t *__restrict__ ncand, uint2 *__restrict__ cand)
{
    __shared__ uint32_t sh_hist[HBINS];
    __shared__ uint32_t sh_sums[HBINS / 4 + 2];
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s0 = (int64_t)blockIdx.x * TK_CHUNK;
    grid_dependency_wait();   // the histograms
    grid_launch_dependents();
    float v[TK_PER];          // this chunk's scores, in flight while the threshold is found
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        const int64_t s = s0 + warp * 32 + j * TK_THREADS + lane;
        v[j] = s < T ? scores[b * T + s] : 0.f;
    }
    const KeyRange r = key_range(keymax[b], nkeymin[b]);
    int dstar;
    uint32_t above;
    find_threshold(hist + (int64_t)b * HBINS, k, sh_hist, sh_sums, &dstar, &above);
    const int64_t nw = (T + 31) >> 5;
    uint32_t *bm = bitmap + b * nw;
    uint2 *cb = cand + (int64_t)b * CAND_CAP;
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        const int base = warp * 32 + j * TK_THREADS;
        const int64_t s = s0 + base + lane;
        bool take = false, isc = false;
        uint32_t key = 0u;
        if (s < T) {
            key = score_key(v[j]);
            const int d = (int)key_digit(key, r);
            take = d > dstar;
            isc = d == dstar;
        }
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (s0 + base < T && lane == 0) bm[(s0 + base) >> 5] = tb;
        const unsigned cb_mask = __ballot_sync(0xffffffffu, isc);
        if (cb_mask != 0u) {
            uint32_t pos0 = 0;
            if (lane == 0) pos0 = atomicAdd(ncand + b, (uint32_t)__popc(cb_mask));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            const uint32_t pos = pos0 + __popc(cb_mask & ((1u << lane) - 1u));
            if (isc && pos < (uint32_t)CAND_CAP) cb[pos] = make_uint2(key, (uint32_t)s);
        }
    }
}

// inclusive scan of one int per thread over the block; *total receives the block sum
__device__ __forceinline__ int block_incl_scan(int v, int *wsum, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) wsum[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int x = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        if (lane < nw) wsum[lane] = x;
    }
    __syncthreads();
    const int before = wid > 0 ? wsum[wid - 1] : 0;
    *total = wsum[nw - 1];
    __syncthreads();
    return v + before;
}

// One CTA per sequence: take the `remaining` best candidates of bin d*, then write the selected
// entries in ascending order from the bitmap (-1 padding when the sequence has fewer than k entries).
__global__ void __launch_bounds__(FIN_THREADS)
topk_final_kernel(const float *__restrict__ scores, int64_t T, int k, const uint32_t *__restrict__ keymax,
                  const uint32_t *__restrict__ nkeymin, const uint32_t *__restrict__ hist, uint32_t *__restrict__ bitmap,
                  const uint32_t *__restrict__ ncand, const uint2 *__restrict__ cand, int32_t *__restrict__ idx)
{
    __shared__ uint32_t sh_hist[HBINS];
    __shared__ uint32_t sh_sums[HBINS / 4 + 2];
    __shared__ uint2 sc[CAND_CAP];
    __shared__ int wsum[32];
    __shared__ uint32_t sh_sel[4];
    const int b = blockIdx.x, tid = threadIdx.x;
    int32_t *out = idx + (int64_t)b * k;
    grid_dependency_wait();   // the candidates and bitmaps (or, without them, the scan)
    grid_launch_dependents();
    if (T <= k) {   // every entry is selected
        for (int j = tid; j < k; j += FIN_THREADS) out[j] = j < T ? j : -1;
        return;
    }
    const KeyRange r = key_range(keymax[b], nkeymin[b]);
    int dstar;
    uint32_t above;
    find_threshold(hist + (int64_t)b * HBINS, k, sh_hist, sh_sums, &dstar, &above);
    const uint32_t remaining = (uint32_t)k - above;
    const int64_t nw = (T + 31) >> 5;
    uint32_t *bm = bitmap + b * nw;
    const uint32_t n = ncand[b];
    if (n <= (uint32_t)CAND_CAP) {
        const uint2 *cb = cand + (int64_t)b * CAND_CAP;
        for (uint32_t i = tid; i < n; i += FIN_THREADS) sc[i] = cb[i];
        __syncthreads();
        for (uint32_t i = tid; i < n; i += FIN_THREADS) {
            const uint2 me = sc[i];
            uint32_t rank = 0;
            for (uint32_t j = 0; j < n; ++j) {
                const uint2 o = sc[j];
                rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
            }
            if (rank < remaining) atomicOr(bm + (me.y >> 5), 1u << (me.y & 31));
        }
    } else {
        // Exact fallback for a crowded threshold bin: radix passes (8 bits) over the keys of bin d*,
        // read from the scores, below the digit; then the keys above the final threshold and the
        // first `remaining` equal ones in index order.
        const float *sq = scores + b * T;
        uint32_t mask = r.dmask == 0u ? 0xffffffffu : ~((1u << r.shift) - 1u);
        uint32_t prefix = r.prefix_hi | ((uint32_t)dstar << r.shift);
        uint32_t rem = remaining;
        int lowbit = r.dmask == 0u ? 0 : r.shift;
        uint32_t *h256 = sh_hist;   // 256 bins
        while (lowbit > 0) {
            const int width = min(8, lowbit), shf = lowbit - width;
            const uint32_t dm = (1u << width) - 1u;
            for (int i = tid; i < 256; i += FIN_THREADS) h256[i] = 0;
            __syncthreads();
            for (int64_t i = tid; i < T; i += FIN_THREADS) {
                const uint32_t key = score_key(sq[i]);
                if ((key & mask) == prefix) atomicAdd(&h256[(key >> shf) & dm], 1u);
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t run = 0;
                int d = 255;
                for (; d > 0; --d) {
                    if (run + h256[d] >= rem) break;
                    run += h256[d];
                }
                sh_sel[0] = (uint32_t)d;
                sh_sel[1] = run;
                sh_sel[2] = h256[d];
            }
            __syncthreads();
            prefix |= sh_sel[0] << shf;
            mask |= dm << shf;
            rem -= sh_sel[1];
            lowbit = shf;
            const bool whole = sh_sel[2] == rem;
            __syncthreads();
            if (whole) break;
        }
        // selection in index order, 1024 entries per round
        int eq_seen = 0;
        for (int64_t base = 0; base < T; base += FIN_THREADS) {
            const int64_t i = base + tid;
            uint32_t key = 0u;
            bool gt = false, eq = false;
            if (i < T) {
                key = score_key(sq[i]);
                gt = (key & mask) > prefix;   // keys of bin d* above the threshold (higher bins are set already)
                eq = (key & mask) == prefix;
            }
            int tot;
            const int rank = block_incl_scan(eq ? 1 : 0, wsum, &tot) - (eq ? 1 : 0);
            const bool sel = gt || (eq && (uint32_t)(eq_seen + rank) < rem);
            if (sel) atomicOr(bm + (i >> 5), 1u << (i & 31));
            eq_seen += tot;
        }
    }
    __syncthreads();
    // write the selected entries in ascending order: each thread a contiguous run of bitmap words
    const int64_t per = (nw + FIN_THREADS - 1) / FIN_THREADS;
    const int64_t w0 = min(nw, (int64_t)tid * per), w1 = min(nw, w0 + per);
    int cnt = 0;
    for (int64_t w = w0; w < w1; ++w) cnt += __popc(bm[w]);
    int total;
    int off = block_incl_scan(cnt, wsum, &total) - cnt;
    for (int64_t w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits != 0u && off < k) {
            const int bit = __ffs(bits) - 1;
            out[off++] = (int32_t)(w * 32 + bit);
            bits &= bits - 1u;
        }
    }
    for (int j = total + tid; j < k; j += FIN_THREADS) out[j] = -1;
}

// ---- the whole top-k of one sequence in one CTA (T <= SEQ_T_MAX) ------------------------------------
//
// The same selection as the three kernels above, on chip: the sequence's keys stay in shared memory,
// so the histogram, the threshold, the collection, the ranking of the threshold bin and the ordered
// output need no global atomics and no further launches.

constexpr int SEQ_T_MAX = 32768;       // 128 KB of keys
constexpr int SEQ_THREADS = 1024;
constexpr int SEQ_SUMS = HBINS / 4 + 4;
constexpr size_t SEQ_SMEM = (size_t)(SEQ_T_MAX + HBINS + SEQ_SUMS + SEQ_T_MAX / 32) * 4 + (size_t)CAND_CAP * 8;

__global__ void __launch_bounds__(SEQ_THREADS, 1)
topk_seq_kernel(const float *__restrict__ scores, int64_t T64, int k, const uint32_t *__restrict__ keymax,
                const uint32_t *__restrict__ nkeymin, int32_t *__restrict__ idx)
{
    extern __shared__ __align__(16) uint32_t seq_sm[];
    uint32_t *skey = seq_sm;                       // [T]
    uint32_t *hist = skey + SEQ_T_MAX;             // [HBINS]
    uint32_t *sums = hist + HBINS;                 // [SEQ_SUMS]
    uint32_t *bm = sums + SEQ_SUMS;                // [T / 32] selection bitmap
    uint2 *cand = reinterpret_cast<uint2 *>(bm + SEQ_T_MAX / 32);   // [CAND_CAP] (key, index)
    __shared__ int wsum[32];
    __shared__ uint32_t sh_sel[4];
    __shared__ uint32_t ncand;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int T = (int)T64;
    int32_t *out = idx + (int64_t)b * k;
    grid_dependency_wait();   // the scores and key ranges of the scan
    grid_launch_dependents();
    if (T <= k) {   // every entry is selected
        for (int j = tid; j < k; j += SEQ_THREADS) out[j] = j < T ? j : -1;
        return;
    }
    const KeyRange r = key_range(keymax[b], nkeymin[b]);
    const int nw = (T + 31) >> 5;
    for (int i = tid; i < HBINS; i += SEQ_THREADS) hist[i] = 0u;
    for (int i = tid; i < nw; i += SEQ_THREADS) bm[i] = 0u;
    if (tid == 0) ncand = 0u;
    __syncthreads();
    // keys into shared memory and the histogram of their digits
    const float *sc = scores + (int64_t)b * T;
    if ((T & 3) == 0) {   // rows 16-byte aligned: all of a thread's scores (up to 32) in flight at once
        float4 v[SEQ_T_MAX / (4 * SEQ_THREADS)];
#pragma unroll
        for (int j = 0; j < SEQ_T_MAX / (4 * SEQ_THREADS); ++j) {
            const int i4 = j * SEQ_THREADS + tid;
            v[j] = 4 * i4 < T ? reinterpret_cast<const float4 *>(sc)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < SEQ_T_MAX / (4 * SEQ_THREADS); ++j) {
            const int i4 = j * SEQ_THREADS + tid;
            if (4 * i4 < T) {
                const uint32_t k0 = score_key(v[j].x), k1 = score_key(v[j].y), k2 = score_key(v[j].z), k3 = score_key(v[j].w);
                reinterpret_cast<uint4 *>(skey)[i4] = make_uint4(k0, k1, k2, k3);
                atomicAdd(&hist[key_digit(k0, r)], 1u);
                atomicAdd(&hist[key_digit(k1, r)], 1u);
                atomicAdd(&hist[key_digit(k2, r)], 1u);
                atomicAdd(&hist[key_digit(k3, r)], 1u);
            }
        }
    } else for (int base = 0; base < T; base += SEQ_THREADS * 8) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * SEQ_THREADS + tid;
            v[j] = i < T ? sc[i] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = base + j * SEQ_THREADS + tid;
            if (i < T) {
                const uint32_t key = score_key(v[j]);
                skey[i] = key;
                atomicAdd(&hist[key_digit(key, r)], 1u);
            }
        }
    }
    __syncthreads();
    int dstar;
    uint32_t above;
    find_threshold(hist, k, hist, sums, &dstar, &above);   // its copy-in reads the histogram in place
    const uint32_t remaining = (uint32_t)k - above;
    // digits above d* are selected (a bitmap bit per entry); digit d* is a candidate
    if ((T & 127) == 0) {
        // four consecutive keys per lane: its nibble of the bitmap, eight lanes per 32-entry word
        for (int i4 = tid; 4 * i4 < T; i4 += SEQ_THREADS) {
            const uint4 kv = reinterpret_cast<const uint4 *>(skey)[i4];
            const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
            uint32_t nib = 0u;
            bool anyc = false;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = (int)key_digit(kk[e], r);
                nib |= (d > dstar ? 1u : 0u) << e;
                anyc |= d == dstar;
            }
            uint32_t word = nib << (4 * (lane & 7));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            word |= __shfl_xor_sync(0xffffffffu, word, 4);
            if ((lane & 7) == 0) bm[i4 >> 3] = word;
            if (__any_sync(0xffffffffu, anyc) && anyc) {   // rare: the threshold bin holds few entries
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if ((int)key_digit(kk[e], r) == dstar) {
                        const uint32_t pos = atomicAdd(&ncand, 1u);
                        if (pos < (uint32_t)CAND_CAP) cand[pos] = make_uint2(kk[e], (uint32_t)(4 * i4 + e));
                    }
            }
        }
    } else for (int base = 0; base < T; base += SEQ_THREADS) {
        const int i = base + tid;
        bool take = false, isc = false;
        uint32_t key = 0u;
        if (i < T) {
            key = skey[i];
            const int d = (int)key_digit(key, r);
            take = d > dstar;
            isc = d == dstar;
        }
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        const int w0 = base + (tid & ~31);
        if (lane == 0 && w0 < T) bm[w0 >> 5] = tb;
        const unsigned cm = __ballot_sync(0xffffffffu, isc);
        if (cm != 0u) {
            uint32_t pos0 = 0;
            if (lane == 0) pos0 = atomicAdd(&ncand, (uint32_t)__popc(cm));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            const uint32_t pos = pos0 + __popc(cm & ((1u << lane) - 1u));
            if (isc && pos < (uint32_t)CAND_CAP) cand[pos] = make_uint2(key, (uint32_t)i);
        }
    }
    __syncthreads();
    const uint32_t n = ncand;
    if (n <= (uint32_t)CAND_CAP) {
        for (uint32_t c = tid; c < n; c += SEQ_THREADS) {
            const uint2 me = cand[c];
            uint32_t rank = 0;
            for (uint32_t j = 0; j < n; ++j) {
                const uint2 o = cand[j];
                rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
            }
            if (rank < remaining) atomicOr(bm + (me.y >> 5), 1u << (me.y & 31));
        }
    } else {
        // Exact fallback for a crowded threshold bin: radix passes (8 bits) over the keys of bin d*
        // below the digit, then the keys above the final threshold and the first `remaining` equal
        // ones in index order.
        uint32_t mask = r.dmask == 0u ? 0xffffffffu : ~((1u << r.shift) - 1u);
        uint32_t prefix = r.prefix_hi | ((uint32_t)dstar << r.shift);
        uint32_t rem = remaining;
        int lowbit = r.dmask == 0u ? 0 : r.shift;
        uint32_t *h256 = hist;
        while (lowbit > 0) {
            const int width = min(8, lowbit), shf = lowbit - width;
            const uint32_t dm = (1u << width) - 1u;
            for (int i = tid; i < 256; i += SEQ_THREADS) h256[i] = 0u;
            __syncthreads();
            for (int i = tid; i < T; i += SEQ_THREADS) {
                const uint32_t key = skey[i];
                if ((key & mask) == prefix) atomicAdd(&h256[(key >> shf) & dm], 1u);
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t run = 0;
                int d = 255;
                for (; d > 0; --d) {
                    if (run + h256[d] >= rem) break;
                    run += h256[d];
                }
                sh_sel[0] = (uint32_t)d;
                sh_sel[1] = run;
                sh_sel[2] = h256[d];
            }
            __syncthreads();
            prefix |= sh_sel[0] << shf;
            mask |= dm << shf;
            rem -= sh_sel[1];
            lowbit = shf;
            const bool whole = sh_sel[2] == rem;
            __syncthreads();
            if (whole) break;
        }
        int eq_seen = 0;
        for (int base = 0; base < T; base += SEQ_THREADS) {
            const int i = base + tid;
            uint32_t key = 0u;
            bool gt = false, eq = false;
            if (i < T) {
                key = skey[i];
                gt = (key & mask) > prefix;   // keys of bin d* above the threshold (higher bins are set already)
                eq = (key & mask) == prefix;
            }
            int tot;
            const int rank = block_incl_scan(eq ? 1 : 0, wsum, &tot) - (eq ? 1 : 0);
            const bool sel = gt || (eq && (uint32_t)(eq_seen + rank) < rem);
            if (sel) atomicOr(bm + (i >> 5), 1u << (i & 31));
            eq_seen += tot;
        }
    }
    __syncthreads();
    // the selected entries in ascending order: each thread a contiguous run of bitmap words
    const int per = (nw + SEQ_THREADS - 1) / SEQ_THREADS;
    const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
    int total;
    int off = block_incl_scan(cnt, wsum, &total) - cnt;
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits != 0u && off < k) {
            const int bit = __ffs(bits) - 1;
            out[off++] = w * 32 + bit;
            bits &= bits - 1u;
        }
    }
    for (int j = total + tid; j < k; j += SEQ_THREADS) out[j] = -1;
}

}  // namespace

// Workspace of the decode index step (256-byte aligned pieces): the head (keymax [B], nkeymin [B]),
// which the caller zeroes before the call; scores [B, T] fp32; a region the scan kernel zeroes (ncand
// [B], hist [B, 2048], bitmap [B, ceil(T/32)]); the candidates [B, 2048] (key, index).
struct DecodeIndexLayout {
    size_t keymax, nkeymin, scores, zero, zero_bytes, ncand, hist, bitmap, cand, total;
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_index_head_bytes(int64_t B) { return al256((size_t)B * 8); }

static DecodeIndexLayout decode_index_layout(int64_t B, int64_t T)
{
    DecodeIndexLayout L;
    L.keymax = 0;
    L.nkeymin = (size_t)B * 4;
    L.scores = decode_index_head_bytes(B);
    L.zero = al256(L.scores + (size_t)B * T * 4);
    L.ncand = L.zero;
    L.hist = al256(L.ncand + (size_t)B * 4);
    L.bitmap = L.hist + (size_t)B * HBINS * 4;
    L.zero_bytes = al256(L.bitmap + (size_t)B * ((T + 31) / 32) * 4) - L.zero;
    L.cand = L.zero + L.zero_bytes;
    L.total = L.cand + (size_t)B * CAND_CAP * 8;
    return L;
}

size_t decode_index_workspace(int64_t B, int64_t T, int k)
{
    (void)k;
    return decode_index_layout(B, T).total + 1024;
}

bool decode_index_tc_supported(int64_t T, int HI, int dI, int k)
{
    return (dI == 64 || dI == 128) && (HI == 16 || HI == 32 || HI == 64 || HI == 128) && T >= 1 && k >= 1 &&
           T <= (1ll << 26);
}

// The top-k after a scan: one CTA per sequence up to SEQ_T_MAX entries, else the chunked kernels;
// each launched as a programmatic dependent of the kernel before it.
static cudaError_t launch_topk_after_scan(char *p8, const DecodeIndexLayout &L, int64_t B, int64_t T, int k, int32_t *idx,
                                          cudaStream_t stream)
{
    float *scores = reinterpret_cast<float *>(p8 + L.scores);
    uint32_t *keymax = reinterpret_cast<uint32_t *>(p8 + L.keymax);
    uint32_t *nkeymin = reinterpret_cast<uint32_t *>(p8 + L.nkeymin);
    uint32_t *ncand = reinterpret_cast<uint32_t *>(p8 + L.ncand);
    uint32_t *hist = reinterpret_cast<uint32_t *>(p8 + L.hist);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(p8 + L.bitmap);
    uint2 *cand = reinterpret_cast<uint2 *>(p8 + L.cand);
    cudaError_t e;
    if (T <= SEQ_T_MAX) {   // the top-k on chip, one CTA per sequence
        if ((e = ensure_smem_limit(reinterpret_cast<const void *>(topk_seq_kernel), SEQ_SMEM)) != cudaSuccess) return e;
        return launch_dependent(topk_seq_kernel, dim3((unsigned)B), dim3(SEQ_THREADS), SEQ_SMEM, stream, (const float *)scores,
                                T, k, (const uint32_t *)keymax, (const uint32_t *)nkeymin, idx);
    }
    if (T > k) {
        const dim3 g2((unsigned)((T + TK_CHUNK - 1) / TK_CHUNK), (unsigned)B);
        e = launch_dependent(topk_hist_kernel, g2, dim3(TK_THREADS), 0, stream, (const float *)scores, T,
                             (const uint32_t *)keymax, (const uint32_t *)nkeymin, hist);
        if (e != cudaSuccess) return e;
        e = launch_dependent(topk_collect_kernel, g2, dim3(TK_THREADS), 0, stream, (const float *)scores, T, k,
                             (const uint32_t *)keymax, (const uint32_t *)nkeymin, (const uint32_t *)hist, bitmap, ncand,
                             cand);
        if (e != cudaSuccess) return e;
    }
    return launch_dependent(topk_final_kernel, dim3((unsigned)B), dim3(FIN_THREADS), 0, stream, (const float *)scores, T,
                            k, (const uint32_t *)keymax, (const uint32_t *)nkeymin, (const uint32_t *)hist, bitmap,
                            (const uint32_t *)ncand, (const uint2 *)cand, idx);
}

// scores/candidates live in `ws` (decode_index_workspace bytes, 256-byte aligned), whose first
// decode_index_head_bytes(B) bytes the caller has zeroed on this stream. The kernels after the scan
// are launched as programmatic dependents, each one scheduled while the one before it finishes.
// Score parameters shared by the bf16 and MXFP4 scans.
static ScoreParams score_params(char *p8, const DecodeIndexLayout &L, const float *w, int64_t B, int64_t T, int HI,
                                int dI, int32_t *status)
{
    ScoreParams sp;
    sp.w = w;
    sp.scores = reinterpret_cast<float *>(p8 + L.scores);
    sp.keymax = reinterpret_cast<uint32_t *>(p8 + L.keymax);
    sp.nkeymin = reinterpret_cast<uint32_t *>(p8 + L.nkeymin);
    sp.status = status;
    sp.zero = reinterpret_cast<uint4 *>(p8 + L.zero);
    sp.zero_n16 = T <= SEQ_T_MAX ? 0 : (int64_t)(L.zero_bytes / 16);   // counters of the chunked top-k
    sp.T = T;
    sp.HI = HI;
    sp.dI = dI;
    sp.tps = (int)((T + BM - 1) / BM);
    sp.G = (int64_t)B * sp.tps;
    sp.stages = 0;
    return sp;
}

cudaError_t launch_decode_index_tc(const uint16_t *qI, const float *w, const uint16_t *kI, int64_t B, int64_t T, int HI,
                                   int dI, int k, int32_t *idx, void *ws, int32_t *status, cudaStream_t stream)
{
    if (B == 0) return cudaSuccess;
    char *p8 = static_cast<char *>(ws);
    const DecodeIndexLayout L = decode_index_layout(B, T);
    CUtensorMap tq, tk;
    if (!make_tmap_bf16_sw128(&tq, qI, (uint64_t)B * HI, dI, HI)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_sw128(&tk, kI, (uint64_t)(B * T), dI, BM)) return cudaErrorInvalidValue;
    ScoreParams sp = score_params(p8, L, w, B, T, HI, dI, status);
    const size_t a_bytes = (size_t)(dI / 64) * BM * 128;
    const size_t fixed = 1024 + 2 * (size_t)(dI / 64) * HI * 128 + 256 * 4 + 256;
    // Two CTAs per SM (two independent tile pipelines) when two stages of each still fit in half of
    // shared memory and the accumulators in half of TMEM; else one CTA with as many stages as fit.
    const size_t half_smem = 113 * 1024;
    const bool two = (int64_t)HI * NACC <= 256 && fixed + 2 * a_bytes <= half_smem;
    sp.stages = (int)std::min<size_t>(MAX_STAGES, ((two ? half_smem : 227 * 1024) - fixed) / a_bytes);
    const size_t smem = fixed + (size_t)sp.stages * a_bytes;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(decode_scores_tc_kernel), smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if ((e = current_device_sms(&dev, &nsm)) != cudaSuccess) return e;
    const unsigned g1 = (unsigned)std::min<int64_t>((two ? 2 : 1) * (int64_t)nsm, sp.G);
    decode_scores_tc_kernel<<<g1, NUM_THREADS, smem, stream>>>(tq, tk, sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_topk_after_scan(p8, L, B, T, k, idx, stream);
}

bool decode_index_fp4_supported(int64_t T, int HI, int dI, int k)
{
    return decode_index_tc_supported(T, HI, dI, k) && (int64_t)T * 4 < (1ll << 31);
}

// MXFP4 operands: codes two per byte (channel 2i in the low nibble), one E8M0 scale per 32 channels.
cudaError_t launch_decode_index_fp4(const uint8_t *qc, const uint8_t *qs, const float *w, const uint8_t *kc,
                                    const uint8_t *ks, int64_t B, int64_t T, int HI, int dI, int k, int32_t *idx,
                                    void *ws, int32_t *status, cudaStream_t stream)
{
    if (B == 0) return cudaSuccess;
    char *p8 = static_cast<char *>(ws);
    const DecodeIndexLayout L = decode_index_layout(B, T);
    CUtensorMap tkc;   // k^I codes as rows of dI/2 bytes, 128-row boxes
    if (!make_tmap_u8_rows(&tkc, kc, (uint64_t)(B * T), (uint64_t)dI / 2, BM)) return cudaErrorInvalidValue;
    if (dI == 128 && HI <= 64 && T % 4 == 0 && (reinterpret_cast<uintptr_t>(qs) & 3u) == 0 &&
        (reinterpret_cast<uintptr_t>(ks) & 15u) == 0 && (reinterpret_cast<uintptr_t>(kc) & 15u) == 0) {
        // block-scaled MMA on the MXFP4 operands as they are
        CUtensorMap tqc;
        if (!make_tmap_u8_sw64(&tqc, qc, (uint64_t)B * HI, (uint32_t)HI)) return cudaErrorInvalidValue;
        Mxf4Params x;
        x.sp = score_params(p8, L, w, B, T, HI, dI, status);
        x.qs = qs;
        x.kc = kc;
        x.ks = ks;
        const size_t smem = 1024 + X4_STAGES * (size_t)X4_A_BYTES + 2 * 4096 + (X4_STAGES + 2) * (size_t)X4_SF_BYTES +
                            256 * 4 + (2 * X4_STAGES + 2 * X4_NACC + 4 + 2) * 8;
        cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(decode_scores_mxf4_kernel), smem);
        if (e != cudaSuccess) return e;
        int dev = 0, nsm = 148;
        if ((e = current_device_sms(&dev, &nsm)) != cudaSuccess) return e;
        const unsigned g1 = (unsigned)std::min<int64_t>(2 * (int64_t)nsm, x.sp.G);   // two CTAs per SM
        decode_scores_mxf4_kernel<<<g1, X4_THREADS, smem, stream>>>(tqc, x);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        return launch_topk_after_scan(p8, L, B, T, k, idx, stream);
    }
    Fp4Params f;
    f.sp = score_params(p8, L, w, B, T, HI, dI, status);
    f.qc = qc;
    f.qs = qs;
    f.ks = ks;
    f.rows = B * T;
    const size_t a_bytes = (size_t)(dI / 64) * BM * 128, b_bytes = (size_t)(dI / 64) * HI * 128;
    const size_t c_bytes = (size_t)dI / 2 * BM;
    const size_t smem = 1024 + 2 * a_bytes + 2 * b_bytes + F4_CST * c_bytes + 256 * 4 + 256 * 4 + 34 * 8;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(decode_scores_fp4_kernel), smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if ((e = current_device_sms(&dev, &nsm)) != cudaSuccess) return e;
    const unsigned g1 = (unsigned)std::min<int64_t>(nsm, f.sp.G);
    decode_scores_fp4_kernel<<<g1, F4_THREADS, smem, stream>>>(tkc, f);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_topk_after_scan(p8, L, B, T, k, idx, stream);
}

}  // namespace csa
