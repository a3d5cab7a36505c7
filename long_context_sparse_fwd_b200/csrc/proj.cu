// proj.cu -- the grouped low-rank output projection after the attention, on the tensor cores.
//
// Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention" (its grouped output
// projection item): the heads are split into o_groups groups; each group's concatenated head outputs
// go through their own o_a_proj to o_lora_rank channels, and the concatenation of all groups goes
// through o_b_proj to hidden_size (llm-atlas "DeepSeek-V4-Flash", config.json table: o_groups 8,
// o_lora_rank 1024, hidden_size 4096). Both steps are GEMMs with K-major operands:
//     z[:, g R:(g+1) R] = o[:, g K:(g+1) K] . Wa[g]^T        (K = (H / G) D, one GEMM per group)
//     out                = z . Wb^T
//
// One persistent kernel serves both: C[M, N] = A[M, K] . B[N, K]^T for G groups, group g reading A
// at column offset g*K, B at row offset g*N and writing C at column offset g*N. Tiles of 128 x 256:
// a 4-deep TMA ring of [128 x 64] A and [256 x 64] B boxes (128-byte swizzle), tcgen05.mma
// M=128 x N=256 x K=16 into one of two TMEM accumulators (2 x 256 columns), and four epilogue warps
// that convert a finished accumulator to bf16 through swizzled staging rows and TMA tensor stores
// while the MMAs of the next tile run. Rows past M are zero-filled on load and clipped on store.
// Every wait is bounded (CSA_ERR_TIMEOUT on expiry).
#include <algorithm>

#include "kernels.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int TM = 128, TN = 256, TK = 64;
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = TM * TK * 2;      // 16 KB
constexpr uint32_t B_BYTES = TN * TK * 2;      // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int EPI_THREADS = 128;
constexpr uint32_t STG_BYTES = 32 * 128;       // one epilogue warp's staging: 32 rows x 64 bf16
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 4 * 2 * STG_BYTES + 256;

// generic-proxy shared-memory writes (the staging rows) made visible to the TMA engine
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

struct ProjParams {
    int32_t *status;
    int64_t M;
    int N, K, G;
    int mt, nt;          // tiles along M and along N (per group)
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
proj_gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_c, ProjParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *stg = smem + (size_t)STAGES * STAGE_BYTES;                 // [4 warps][2][STG_BYTES]
    uint64_t *bars = reinterpret_cast<uint64_t *>(stg + 4 * 2 * STG_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES, *tfull = bars + 2 * STAGES, *tempty = bars + 2 * STAGES + 2;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 2 * STAGES + 5);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles = (int64_t)p.G * p.mt * p.nt;
    const int ksteps = p.K / TK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
        }
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    // tile t: n fastest (consecutive CTAs share the A rows), then m, then the group
    auto tile_coords = [&](int64_t t, int &g, int &m, int &n) {
        n = (int)(t % p.nt);
        const int64_t r = t / p.nt;
        m = (int)(r % p.mt);
        g = (int)(r / p.mt);
    };

    if (warp == 0) {
        // ---------------- TMA producer (warp-wide loop, one elected lane issues) ----------------
        if (elect_one()) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
        }
        int it = 0;   // stage uses so far
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            int g, m, n;
            tile_coords(t, g, m, n);
            for (int k = 0; k < ksteps; ++k, ++it) {
                const int st = it % STAGES;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((it / STAGES) & 1) ^ 1, abort, p.status))) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    uint8_t *sa = smem + (size_t)st * STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
                    tma_load_2d(sa, &tm_a, &full[st], g * p.K + k * TK, m * TM);
                    tma_load_2d(sa + A_BYTES, &tm_b, &full[st], k * TK, g * p.N + n * TN);
                }
                __syncwarp();
            }
        }
        // never leave with copies in flight into this CTA's shared memory
        for (int i = max(0, it - STAGES); i < it; ++i)
            mbar_wait(&full[i % STAGES], (i / STAGES) & 1, abort, p.status, 100000000ull);
    } else if (warp == 1) {
        // ---------------- MMA issuer (warp-wide loop, one elected lane issues) ----------------
        const uint32_t idesc = idesc_bf16(TM, TN);
        const uint64_t d0 = sdesc_sw128(smem_u32(smem), 16, 1024);
        int it = 0, tc = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
            const int buf = tc & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((tc >> 1) & 1) ^ 1, abort, p.status))) break;
            tc_fence_after();
            for (int k = 0; k < ksteps; ++k, ++it) {
                const int st = it % STAGES;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (it / STAGES) & 1, abort, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
                    const uint64_t da = d0 + (((uint32_t)st * STAGE_BYTES) >> 4);
                    const uint64_t db = d0 + (((uint32_t)st * STAGE_BYTES + A_BYTES) >> 4);
#pragma unroll
                    for (int ks = 0; ks < TK / 16; ++ks)
                        mma_bf16(tmem + buf * TN, da + 2 * ks, db + 2 * ks, idesc, (k | ks) != 0);
                    mma_commit(&empty[st]);
                    if (k + 1 == ksteps) mma_commit(&tfull[buf]);
                }
                __syncwarp();
            }
        }
        // TMEM is released after the final barrier: wait (bounded) until the last accumulator is complete
        if (tc > 0) mbar_wait(&tfull[(tc - 1) & 1], ((tc - 1) >> 1) & 1, abort, p.status, 100000000ull);
        __syncwarp();
    } else {
        // ---------------- epilogue: TMEM -> bf16 -> staging rows -> TMA tensor stores ----------------
        const int q = warp & 3;                               // TMEM lanes 32q .. 32q+31 = tile rows
        uint8_t *mystg = stg + (size_t)(warp - 2) * 2 * STG_BYTES;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        int tc = 0, nst = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
            int g, m, n;
            tile_coords(t, g, m, n);
            const int buf = tc & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (tc >> 1) & 1, abort, p.status))) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < TN / 64; ++c, ++nst) {
                float v0[32], v1[32];
                tmem_ld32(trow + buf * TN + c * 64, v0);
                tmem_ld32(trow + buf * TN + c * 64 + 32, v1);
                tmem_wait_ld();
                if (c == TN / 64 - 1) {
                    tc_fence_before();
                    mbar_arrive(&tempty[buf]);   // the accumulator may take the next tile's MMAs
                }
                uint8_t *sb = mystg + (nst & 1) * STG_BYTES;
                // this buffer's previous store must have finished reading it
                if (elect_one()) bulk_wait_read_le1();
                __syncwarp();
                uint8_t *row = sb + lane * 128;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4 *>(row + ((u ^ (lane & 7)) << 4)) =
                        make_uint4(pack_bf2(v0[8 * u], v0[8 * u + 1]), pack_bf2(v0[8 * u + 2], v0[8 * u + 3]),
                                   pack_bf2(v0[8 * u + 4], v0[8 * u + 5]), pack_bf2(v0[8 * u + 6], v0[8 * u + 7]));
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint4 *>(row + (((u + 4) ^ (lane & 7)) << 4)) =
                        make_uint4(pack_bf2(v1[8 * u], v1[8 * u + 1]), pack_bf2(v1[8 * u + 2], v1[8 * u + 3]),
                                   pack_bf2(v1[8 * u + 4], v1[8 * u + 5]), pack_bf2(v1[8 * u + 6], v1[8 * u + 7]));
                fence_async_smem();
                __syncwarp();
                if (elect_one()) {
                    tma_store_2d(&tm_c, sb, g * p.N + n * TN + c * 64, (int)(m * TM + q * 32));
                    bulk_commit();
                }
                __syncwarp();
            }
        }
        if (elect_one()) bulk_wait_all();   // every store of this warp has completed
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool proj_gemm_tc_supported(int64_t M, int N, int K, int G)
{
    return M >= 1 && M < (1ll << 31) && N >= TN && N % TN == 0 && K >= TK && K % TK == 0 && G >= 1 &&
           (int64_t)G * N < (1ll << 31) && (int64_t)G * K < (1ll << 31);
}

// C[:, g N:(g+1) N] = A[:, g K:(g+1) K] . B[g N:(g+1) N, :]^T for g < G; A [M, lda], B [G N, K], C [M, ldc], bf16.
cudaError_t launch_proj_gemm_tc(const uint16_t *A, int64_t lda, const uint16_t *B, uint16_t *C, int64_t ldc, int64_t M,
                                int N, int K, int G, int32_t *status, cudaStream_t stream)
{
    if (M == 0) return cudaSuccess;
    CUtensorMap ta, tb, tcm;
    if (!make_tmap_bf16_sw128(&ta, A, (uint64_t)M, (uint64_t)lda, TM)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_sw128(&tb, B, (uint64_t)G * N, (uint64_t)K, TN)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_sw128(&tcm, C, (uint64_t)M, (uint64_t)ldc, 32)) return cudaErrorInvalidValue;
    ProjParams p;
    p.status = status;
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = G;
    p.mt = (int)((M + TM - 1) / TM);
    p.nt = N / TN;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(proj_gemm_tc_kernel), SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if ((e = current_device_sms(&dev, &sms)) != cudaSuccess) return e;
    const int64_t tiles = (int64_t)G * p.mt * p.nt;
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, sms);
    proj_gemm_tc_kernel<<<grid, NUM_THREADS, SMEM, stream>>>(ta, tb, tcm, p);
    return cudaGetLastError();
}

}  // namespace csa
