// attend_tc.cu -- CSA / HCA prefill attention on the 5th-generation tensor cores (H=64, D=512,
// rope 64), one query per CTA.
//
// What it computes (Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention":
// shared K=V MQA, partial interleaved RoPE with the output rope slice rotated at -i (eq. 26), a
// per-head sink (eq. 27), the sliding-window branch concatenated with the compressed entries;
// section "Attention mask layout": window (i - W, i], CSA picks from the indexer, HCA every
// entry w < (i+1)//m): for query t and head h, one softmax over the window rows kv_rot[j]
// (scored with q rotated by theta_tok) and the entry rows C[s] (scored with q rotated by
// theta_cmp) plus exp(sink_h); K = V; each branch's rope slice rotated back by -t with its theta.
//
// Design. A query's 64 heads form an M=64 tile; its keys (window rows first, then the entries)
// are gathered 64 at a time with 16-byte cp.async into 128-byte-swizzled shared memory, where the
// same tile is the K-major B operand of S = Q K^T and the MN-major B operand of O += P V:
// the selected rows are read from L2/HBM once and shared by all 64 heads.
//   TMEM (M=64 uses 16 lanes of each 32-lane quarter; a second tile sits at lane offset 16):
//     lanes +0 : O_lo  cols [0,256)   output dims 0..255
//     lanes +16: O_hi  cols [0,192)   dims 256..447, cols [192,256) entry-branch rope dims 448..511
//     lanes +16: O_rw  cols [256,320) window-branch rope dims 448..511
//     S_b      cols [320,384) at lanes +16*(b&1)    (double-buffered logits)
//   The rope slice of each branch accumulates separately so each can be rotated back by -t
//   with its own theta in the epilogue.
// Softmax runs in the exp2 domain with a reference max per head that is only raised when a block
// exceeds it by more than 2^8 (then O is rescaled in TMEM after the previous P V completes),
// so almost every block needs no rescale. The sink seeds the reference and the running sum.
// Keys arrive by 16-byte cp.async from four loader warps (each row 1 KB, two 512-byte coalesced
// halves per warp instruction), written straight into the swizzled layout.
// The epilogue transposes each warp's output tile through shared memory into 128-byte row segments.
// Roles: warps 0-3 softmax + epilogue, warps 4-7 load keys, warp 8 owns TMEM and issues MMAs
// from an event loop (a P V never waits for the next block's keys).
// Every wait is bounded (CSA_ERR_TIMEOUT on expiry).
#include <algorithm>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int HH = 64, DD = 512, RR = 64;
constexpr int KB = 64;                          // keys per block
constexpr int NCH = DD / 64;                    // 64-element chunks per row
constexpr int QCH = 9;                          // Q chunks: 7 un-rotated, rope(theta_cmp), rope(theta_tok)
constexpr int QCHUNK = HH * 128;                // 8 KB
constexpr int KCHUNK = KB * 128;                // 8 KB
constexpr int STAGE = NCH * KCHUNK;             // 64 KB
constexpr int PBUF = HH * 128;                  // 8 KB
constexpr int NUM_THREADS = 288;
constexpr int SM_THREADS = 128;
constexpr int LOAD_WARP0 = 4;                   // warps 4..7 load keys
constexpr int LOAD_THREADS = 128;
constexpr int MMA_WARP = 8;
constexpr float TAU = 8.f;
constexpr uint32_t COL_RW = 256, COL_S = 320;
constexpr uint32_t LANE16 = 16u << 16;
constexpr uint32_t TMEM_COLS = 512;


constexpr size_t OFF_Q = 0;
constexpr size_t OFF_KV = OFF_Q + (size_t)QCH * QCHUNK;       // 72 KB
constexpr size_t OFF_P = OFF_KV + 2 * (size_t)STAGE;          // 200 KB
constexpr size_t OFF_ROPE = OFF_P + 2 * (size_t)PBUF;         // 216 KB: cos/sin [2 thetas][32 pairs][2]
constexpr size_t OFF_BAR = OFF_ROPE + 2 * 32 * 2 * 4;
constexpr size_t OFF_LIST = OFF_BAR + 256;

struct TcArgs {
    const uint16_t *q;        // [R, 64, 512] (R = S prefill rows or B decode sequences)
    const uint16_t *kv_rot;   // prefill: [S, 512] window rows; decode: [B, W, 512] (positions P-W+1..P)
    const uint16_t *C;        // prefill: [T, 512]; decode: [B, T, 512] bf16 (or null: FP8 cache)
    const uint8_t *c8;        // decode FP8 cache: [B, T, 448] E4M3 codes
    const float *c8_scale;    //                   [B, T]
    const uint16_t *c_rope;   //                   [B, T, 64] bf16
    const int32_t *idx;       // [R, k] or null (HCA: every visible entry)
    const float *sinks;       // [64]
    float *o;                 // [R, 64, 512]
    float *part_ml;           // split partials: [R*nsplit, 64, 2] (log2-domain reference max, sum)
    int32_t *status;
    int64_t S, T, P;          // S: prefill rows; P: decode position
    int k, W, m, decode, nsplit;
    float scale_log2;         // softmax scale * log2(e)
    double log2_theta_tok, log2_theta_cmp;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// arrive on `bar` when this thread's earlier cp.async copies have landed (no pending-count increment)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// byte offset of 16-byte unit `u` (0..7) of row `row` inside a 128-byte-swizzled [rows x 128 B] chunk
__device__ __forceinline__ uint32_t sw128(int row, int u) { return (uint32_t)(row * 128 + ((u ^ (row & 7)) << 4)); }

__global__ void __launch_bounds__(NUM_THREADS, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, TcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = smem + OFF_Q;
    uint8_t *sKV = smem + OFF_KV;
    uint8_t *sP = smem + OFF_P;
    float *rope_cs = reinterpret_cast<float *>(smem + OFF_ROPE);     // [theta: 0 tok, 1 cmp][pair][cos, sin]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *kv_full = bars + 0;     // [2] loader arrivals
    uint64_t *kv_empty = bars + 2;    // [2] MMA commit
    uint64_t *s_full = bars + 4;      // [2] MMA commit
    uint64_t *p_ready = bars + 6;     // [2] 128 softmax arrivals
    // P V completion: block b commits o_done[b & 1]. When the softmax of block b waits for P V of
    // block b-1, every earlier completion of that barrier (block b-3) is already known to be done
    // (it preceded S of block b), so a parity wait cannot mistake an older phase for the one wanted.
    uint64_t *o_done = bars + 8;      // [2]
    uint64_t *o_final = bars + 10;    // single use: every MMA of this CTA has completed
    uint64_t *q_ready = bars + 11;    // 128 softmax arrivals
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 12);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 13);
    int *nlist = reinterpret_cast<int *>(bars + 14);
    uint64_t *q_tma = bars + 15;      // TMA of the 7 un-rotated Q chunks
    int *elist = reinterpret_cast<int *>(smem + OFF_LIST);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // prefill: one CTA per query row, longest key lists first; decode: nsplit CTAs per sequence
    const int64_t row = a.decode ? (int64_t)(blockIdx.x / a.nsplit) : a.S - 1 - (int64_t)blockIdx.x;
    const int split = a.decode ? (int)(blockIdx.x % a.nsplit) : 0;
    const bool partial = a.nsplit > 1;
    const int64_t t = a.decode ? a.P : row;                   // position of the query
    const int64_t vis = a.decode ? a.T : visible_entries(t, a.m, a.T);
    const int64_t wpos0 = max((int64_t)0, t - a.W + 1);
    const int nw = (int)(t - wpos0 + 1);
    const uint16_t *win0 = a.decode ? a.kv_rot + (row * a.W + (a.W - nw)) * (int64_t)DD
                                    : a.kv_rot + wpos0 * (int64_t)DD;   // first window row
    const uint16_t *ent0 = a.decode && a.C != nullptr ? a.C + row * a.T * DD : a.C;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kv_full[i], LOAD_THREADS);   // one cp.async arrival per loader thread
            mbar_init(&kv_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_ready[i], SM_THREADS);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(o_final, 1);
        mbar_init(q_ready, SM_THREADS);
        mbar_init(q_tma, 1);
        *abort = 0;
        fence_barrier_init();
        mbar_arrive_expect_tx(q_tma, 7 * QCHUNK);
        const uint64_t pol_q = policy_evict_first();     // q is read once
        for (int dc = 0; dc < 7; ++dc) tma_load_2d_hint(sQ + dc * QCHUNK, &tm_q, q_tma, dc * 64, (int)(row * HH), pol_q);
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_ptr, TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x < 64) {   // rope table: angle t * theta^(-2p/64) for both thetas
        const int p = threadIdx.x & 31, th = threadIdx.x >> 5;
        float c, s;
        rope_cos_sin((double)t, p, RR, th ? a.log2_theta_cmp : a.log2_theta_tok, &c, &s);
        rope_cs[(th * 32 + p) * 2] = c;
        rope_cs[(th * 32 + p) * 2 + 1] = s;
    }
    if (warp == LOAD_WARP0) { // compacted entry list (CSA); HCA uses entries 0..vis-1 directly
        if (a.idx != nullptr) {
            const int32_t *ir = a.idx + row * (int64_t)a.k;
            int vals[32];   // k <= 1024: all loads in flight at once
#pragma unroll
            for (int i = 0; i < 32; ++i) vals[i] = i * 32 + lane < a.k ? __ldg(ir + i * 32 + lane) : -1;
            int cnt = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int s = vals[i];
                const bool ok = s >= 0 && (int64_t)s < vis;
                if (s >= 0 && !ok) report(a.status, CSA_ERR_INVALID_ARG);
                const unsigned mk = __ballot_sync(0xffffffffu, ok);
                if (ok) elist[cnt + __popc(mk & ((1u << lane) - 1u))] = s;
                cnt += __popc(mk);
            }
            if (lane == 0) *nlist = cnt;
        } else if (lane == 0) {
            *nlist = (int)vis;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const int ne = *nlist;
    const int nbw = (nw + KB - 1) / KB, nbe = (ne + KB - 1) / KB, nb_all = nbw + nbe;
    // this CTA's share of the key blocks (window blocks first, then entry blocks)
    const int gb0 = (int)((int64_t)split * nb_all / a.nsplit);
    const int nb = (int)((int64_t)(split + 1) * nb_all / a.nsplit) - gb0;
    const bool has_win = gb0 < nbw && nb > 0, has_ent = gb0 + nb > nbw;

    if (warp < 4) {
        // =============== softmax + epilogue (warp w owns TMEM lane quarter w) ===============
        const int tid = threadIdx.x;
        // Q tile: 7 un-rotated chunks, rope chunk rotated with theta_cmp (7) and theta_tok (8)
        uint4 qv[4];   // rope chunk: 64 heads x 8 units, 4 per thread, all loads in flight
#pragma unroll
        for (int r4 = 0; r4 < 4; ++r4) {
            const int i = tid + r4 * SM_THREADS, h = i >> 3, uu = i & 7;
            qv[r4] = __ldg(reinterpret_cast<const uint4 *>(a.q + ((row * HH + h) * (int64_t)DD) + 448 + uu * 8));
        }
#pragma unroll
        for (int r4 = 0; r4 < 4; ++r4) {
            const int i = tid + r4 * SM_THREADS, h = i >> 3, uu = i & 7;
            const uint4 v = qv[r4];
            {
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                uint32_t oc[4], ot[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int p = uu * 4 + e;
                    const float x0 = bf_lo(w4[e]), x1 = bf_hi(w4[e]);
                    const float cc = rope_cs[(32 + p) * 2], sc = rope_cs[(32 + p) * 2 + 1];
                    const float ct = rope_cs[p * 2], st = rope_cs[p * 2 + 1];
                    oc[e] = pack_bf2(x0 * cc - x1 * sc, x0 * sc + x1 * cc);
                    ot[e] = pack_bf2(x0 * ct - x1 * st, x0 * st + x1 * ct);
                }
                *reinterpret_cast<uint4 *>(sQ + 7 * QCHUNK + sw128(h, uu)) = make_uint4(oc[0], oc[1], oc[2], oc[3]);
                *reinterpret_cast<uint4 *>(sQ + 8 * QCHUNK + sw128(h, uu)) = make_uint4(ot[0], ot[1], ot[2], ot[3]);
            }
        }
        fence_async_smem();
        mbar_arrive(q_ready);

        const int h = warp * 16 + (lane & 15);
        const int half = lane >> 4;
        // the sink seeds the running max and sum; split partials leave it to the combine step
        const float zl = partial ? -INFINITY : a.sinks[h] * 1.4426950408889634f;
        float m_ref = zl, l = (zl == -INFINITY) ? 0.f : 1.f;
        const uint32_t tq = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        for (int b = 0; b < nb && ok; ++b) {
            const int buf = b & 1;
            const int gb = gb0 + b;
            const int nk = gb < nbw ? min(KB, nw - gb * KB) : min(KB, ne - (gb - nbw) * KB);
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (b >> 1) & 1, abort, a.status));
            if (!ok) break;
            tc_fence_after();
            float s0[32], s1[32];
            tmem_ld32(tq + COL_S, s0);
            tmem_ld32(tq + COL_S + 32, s1);
            tmem_wait_ld();
            const bool active = half == buf;
            float corr = 1.f;
            bool need = false;
            if (active) {
                float mb = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s0[j] = j < nk ? s0[j] * a.scale_log2 : -INFINITY;
                    s1[j] = j + 32 < nk ? s1[j] * a.scale_log2 : -INFINITY;
                    mb = fmaxf(mb, fmaxf(s0[j], s1[j]));
                }
                if (mb > m_ref + TAU) {
                    corr = exp2f(m_ref - mb);
                    m_ref = mb;
                    l *= corr;
                    need = b > 0;
                }
                float sum = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const uint32_t w0 = pack_bf2(exp2f(s0[j] - m_ref), exp2f(s0[j + 1] - m_ref));
                    const uint32_t w1 = pack_bf2(exp2f(s1[j] - m_ref), exp2f(s1[j + 1] - m_ref));
                    pk[j >> 1] = w0;
                    pk[16 + (j >> 1)] = w1;
                    sum += bf_lo(w0) + bf_hi(w0) + bf_lo(w1) + bf_hi(w1);
                }
                l += sum;
                uint8_t *prow = sP + buf * PBUF;
#pragma unroll
                for (int uu = 0; uu < 8; ++uu)
                    *reinterpret_cast<uint4 *>(prow + sw128(h, uu)) =
                        make_uint4(pk[uu * 4], pk[uu * 4 + 1], pk[uu * 4 + 2], pk[uu * 4 + 3]);
            }
            // keep both halves of the warp in step: the partner lane holds the same head
            const float pm = __shfl_xor_sync(0xffffffffu, m_ref, 16);
            const float pl = __shfl_xor_sync(0xffffffffu, l, 16);
            const float pc = __shfl_xor_sync(0xffffffffu, corr, 16);
            const int pn = __shfl_xor_sync(0xffffffffu, (int)need, 16);
            if (!active) { m_ref = pm; l = pl; corr = pc; need = pn != 0; }
            if (__any_sync(0xffffffffu, need)) {
                // O must hold every earlier P V before it is rescaled
                ok = __all_sync(0xffffffffu, mbar_wait(&o_done[(b - 1) & 1], ((b - 1) >> 1) & 1, abort, a.status));
                tc_fence_after();
                if (ok) {
                    for (uint32_t c = 0; c < COL_S; c += 32) {
                        float v[32];
                        tmem_ld32(tq + c, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= corr;
                        tmem_st32(tq + c, v);
                    }
                    tmem_wait_st();
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&p_ready[buf]);
        }
        // ---------------- epilogue ----------------
        if (ok && nb > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_final, 0, abort, a.status));
        if (ok && nb > 0) {
            tc_fence_after();
            const float inv = partial ? 1.f : (l > 0.f ? 1.f / l : 0.f);
            // Every MMA has completed, so the P buffers are idle: each warp transposes its 32 rows x 32
            // columns (16 heads x two dim halves) through its own 4 KB slice and writes whole 128-byte
            // row segments (8 lanes per segment) to the output.
            uint8_t *wbuf = sP + warp * 4096;
            float *obase = partial ? a.o + ((row * a.nsplit + split) * HH) * (int64_t)DD   // o = partial rows
                                   : a.o + (row * HH) * (int64_t)DD;
            for (int c = 0; c < 256; c += 32) {
                float v[32], rw[32];
                tmem_ld32(tq + c, v);
                if (c >= 192) tmem_ld32(tq + COL_RW + (c - 192), rw);   // warp-uniform collective loads
                tmem_wait_ld();
                if (half == 1 && c >= 192) {
                    // rope slice: entry branch (here) + window branch (O_rw), each rotated by -t
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const int p = (c - 192 + j) >> 1;
                        const float ct = rope_cs[p * 2], st = rope_cs[p * 2 + 1];
                        const float cc = rope_cs[(32 + p) * 2], sc = rope_cs[(32 + p) * 2 + 1];
                        float e0 = has_ent ? v[j] : 0.f, e1 = has_ent ? v[j + 1] : 0.f;
                        float w0 = has_win ? rw[j] : 0.f, w1 = has_win ? rw[j + 1] : 0.f;
                        v[j] = (e0 * cc + e1 * sc) + (w0 * ct + w1 * st);
                        v[j + 1] = (-e0 * sc + e1 * cc) + (-w0 * st + w1 * ct);
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4 *>(wbuf + sw128(lane, u)) =
                        make_float4(v[4 * u] * inv, v[4 * u + 1] * inv, v[4 * u + 2] * inv, v[4 * u + 3] * inv);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int pr = i * 4 + (lane >> 3), u = lane & 7;   // row pr of this warp's tile
                    const float4 x = *reinterpret_cast<const float4 *>(wbuf + sw128(pr, u));
                    const int hh = warp * 16 + (pr & 15);
                    __stcs(reinterpret_cast<float4 *>(obase + hh * (int64_t)DD + (pr >> 4) * 256 + c + u * 4), x);
                }
                __syncwarp();
            }
        } else if (nb == 0 && !partial) {
            float *orow = a.o + ((row * HH + h) * (int64_t)DD) + half * 256;
            for (int c = 0; c < 256; c += 4) *reinterpret_cast<float4 *>(orow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (partial && lane < 16) {   // reference max (log2 domain) and sum of this split; an empty split has l = 0
            float *ml = a.part_ml + ((row * a.nsplit + split) * HH + h) * 2;
            ml[0] = ok && nb > 0 ? m_ref : -INFINITY;
            ml[1] = ok && nb > 0 ? l : 0.f;
        }
    } else if (warp >= LOAD_WARP0 && warp < MMA_WARP) {
        // =============== key loads: 16-byte cp.async into the swizzled stages ===============
        const int lw = warp - LOAD_WARP0;        // rows 16*lw .. 16*lw+15 of each block
        for (int b = 0; b < nb; ++b) {
            const int st = b & 1, gb = gb0 + b;
            if (!__all_sync(0xffffffffu, mbar_wait(&kv_empty[st], ((b >> 1) & 1) ^ 1, abort, a.status))) break;
            const bool win = gb < nbw;
            const int kbase = win ? gb * KB : (gb - nbw) * KB;
            const int nk = win ? min(KB, nw - kbase) : min(KB, ne - kbase);
            if (!win && a.C == nullptr) {
                // FP8 entry cache: codes * per-entry scale on channels [0,448), bf16 rope on [448,512),
                // converted to bf16 here and stored into the swizzled stage
                uint8_t *stage = sKV + st * STAGE;
#pragma unroll 2
                for (int r = 0; r < 16; ++r) {
                    const int key = lw * 16 + r;
                    uint4 o0 = make_uint4(0u, 0u, 0u, 0u), o1 = o0;
                    if (key < nk) {
                        const int64_t e = row * a.T + (a.idx != nullptr ? elist[kbase + key] : kbase + key);
                        if (lane < 28) {
                            const float sc = __ldg(a.c8_scale + e);
                            const uint4 cv = __ldg(reinterpret_cast<const uint4 *>(a.c8 + e * 448) + lane);
                            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
                            uint32_t ow[8];
#pragma unroll
                            for (int q2 = 0; q2 < 8; ++q2) {
                                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                                    (__nv_fp8x2_storage_t)((cw[q2 >> 1] >> ((q2 & 1) * 16)) & 0xffffu), __NV_E4M3);
                                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
                                ow[q2] = pack_bf2(f.x * sc, f.y * sc);
                            }
                            o0 = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                            o1 = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                        } else {
                            const uint4 *rr = reinterpret_cast<const uint4 *>(a.c_rope + e * 64);
                            o0 = __ldg(rr + 2 * (lane - 28));
                            o1 = __ldg(rr + 2 * (lane - 28) + 1);
                        }
                    }
                    // lane < 28: dims [16*lane, 16*lane+16); lanes 28..31: rope dims 448 + 16*(lane-28)
                    const int d0 = lane < 28 ? 16 * lane : 448 + 16 * (lane - 28);
                    const int dc = d0 >> 6, u0 = (d0 & 63) >> 3;
                    *reinterpret_cast<uint4 *>(stage + dc * KCHUNK + sw128(key, u0)) = o0;
                    *reinterpret_cast<uint4 *>(stage + dc * KCHUNK + sw128(key, u0 + 1)) = o1;
                }
                fence_async_smem();
                mbar_arrive(&kv_full[st]);
                continue;
            }
            const uint32_t sbase = smem_u32(sKV + st * STAGE);
#pragma unroll 4
            for (int r = 0; r < 16; ++r) {
                const int key = lw * 16 + r;
                const bool valid = key < nk;
                const uint16_t *rowp = a.q;      // any mapped address for padding rows (zero-filled, 0 bytes read)
                if (valid) {
                    if (win) rowp = win0 + (int64_t)(kbase + key) * DD;
                    else rowp = ent0 + (int64_t)(a.idx != nullptr ? elist[kbase + key] : kbase + key) * DD;
                }
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    const int u = lane + 32 * hlf;
                    cp_async16(sbase + (u >> 3) * KCHUNK + sw128(key, u & 7), rowp + (valid ? u * 8 : 0), valid ? 16u : 0u);
                }
            }
            cp_async_arrive_noinc(&kv_full[st]);
        }
        cp_async_wait_all();   // never leave with copies in flight into this CTA's shared memory
    } else if (warp == MMA_WARP && lane == 0) {
        // =============== MMA issuer: one thread, event loop ===============
        const uint32_t idS = idesc_bf16(64, 64);
        const uint32_t idPV256 = idesc_bf16(64, 256, true);
        const uint32_t idPV192 = idesc_bf16(64, 192, true);
        const uint32_t idPV64 = idesc_bf16(64, 64, true);
        // descriptors are formed once; a tile / k-step offset is added to the start-address field
        const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t dK = sdesc_sw128(smem_u32(sKV), 16, 1024);
        const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);
        const uint64_t dV = sdesc_sw128(smem_u32(sKV), KCHUNK, 1024);
        int nS = 0, nPV = 0;
        bool ok = nb == 0 || (mbar_wait(q_ready, 0, abort, a.status) && mbar_wait(q_tma, 0, abort, a.status));
        uint64_t t_progress = globaltimer();
        uint32_t polls = 0;
        while (ok && nPV < nb) {
            bool progressed = false;
            // S(nS) needs its keys and a free logits buffer (softmax of nS-2 finished, i.e. PV(nS-2) issued)
            if (nS < nb && nS <= nPV + 1 && mbar_try_wait(&kv_full[nS & 1], (nS >> 1) & 1)) {
                fence_async_smem();   // keys were written by cp.async (generic proxy); the MMA reads via the async proxy
                tc_fence_after();
                const int st = nS & 1;
                const uint32_t d = tmem + COL_S + (uint32_t)st * LANE16;
                const int rope_chunk = gb0 + nS < nbw ? 8 : 7;
                for (int dc = 0; dc < NCH; ++dc) {
                    const uint64_t qa = dQ + (((dc < 7 ? dc : rope_chunk) * QCHUNK) >> 4);
                    const uint64_t kb = dK + ((st * STAGE + dc * KCHUNK) >> 4);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) mma_bf16(d, qa + 2 * ks, kb + 2 * ks, idS, (dc | ks) != 0);
                }
                mma_commit(&s_full[st]);
                ++nS;
                progressed = true;
            }
            // PV(nPV) needs the softmax of block nPV
            if (nPV < nS && mbar_try_wait(&p_ready[nPV & 1], (nPV >> 1) & 1)) {
                tc_fence_after();
                const int b = nPV, st = b & 1, gb = gb0 + b;
                const bool win = gb < nbw;
                const uint32_t drope = win ? tmem + LANE16 + COL_RW : tmem + LANE16 + 192;
                // the first block of each branch handled by this CTA starts that branch's rope accumulator
                const bool rope_first = win ? (b == 0) : (gb == max(nbw, gb0));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = dP + ((st * PBUF + ks * 32) >> 4);
                    const uint64_t vb = dV + ((st * STAGE + ks * 2048) >> 4);
                    mma_bf16(tmem, ad, vb, idPV256, b > 0 || ks > 0);                                  // dims 0..255
                    mma_bf16(tmem + LANE16, ad, vb + ((4 * KCHUNK) >> 4), idPV192, b > 0 || ks > 0);   // 256..447
                    mma_bf16(drope, ad, vb + ((7 * KCHUNK) >> 4), idPV64, !rope_first || ks > 0);     // 448..511
                }
                mma_commit(&kv_empty[st]);
                mma_commit(&o_done[b & 1]);
                if (b + 1 == nb) mma_commit(o_final);
                ++nPV;
                progressed = true;
            }
            if (progressed) {
                t_progress = globaltimer();
            } else if ((++polls & 255u) == 0) {
                if (*abort) { ok = false; break; }
                if (globaltimer() - t_progress > 2000000000ull) {
                    *abort = 1;
                    report(a.status, CSA_ERR_TIMEOUT);
                    ok = false;
                }
            }
        }
        // leave only when every issued MMA has completed
        mbar_wait(q_tma, 0, abort, a.status, 100000000ull);
        if (nPV == nb && nb > 0) {
            mbar_wait(o_final, 0, abort, a.status, 100000000ull);
        } else if (nS > 0 || nPV > 0) {
            // stopped early: commit once more and wait for that (covers every MMA issued so far)
            mma_commit(o_final);
            mbar_wait(o_final, 0, abort, a.status, 100000000ull);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

bool attend_tc_supported(int H, int D, int r, int k)
{
    return H == HH && D == DD && r == RR && k <= 1024;
}

// Combine the split partials of decode: per (sequence, head), o = sum_i 2^(m_i - M) O_i / L with
// L = 2^(z - M) + sum_i 2^(m_i - M) l_i and M the largest of the split maxima and the sink z (all in
// the log2 domain). The sink enters here exactly once.
__global__ void __launch_bounds__(128)
combine_splits_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml, const float *__restrict__ sinks,
                      int nsplit, float *__restrict__ o)
{
    const int64_t b = blockIdx.x / HH;
    const int h = blockIdx.x % HH;
    const float z = sinks[h] * 1.4426950408889634f;
    float M = z;
    for (int i = 0; i < nsplit; ++i) {
        const float mi = part_ml[((b * nsplit + i) * HH + h) * 2];
        M = fmaxf(M, mi);
    }
    float L = (z == -INFINITY) ? 0.f : exp2f(z - M);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < nsplit; ++i) {
        const float mi = part_ml[((b * nsplit + i) * HH + h) * 2];
        const float li = part_ml[((b * nsplit + i) * HH + h) * 2 + 1];
        if (mi == -INFINITY || li == 0.f) continue;   // empty split: its O was never written
        const float wgt = exp2f(mi - M);
        L += wgt * li;
        const float4 v = reinterpret_cast<const float4 *>(part_o + ((b * nsplit + i) * HH + h) * (int64_t)DD)[threadIdx.x];
        acc.x += wgt * v.x;
        acc.y += wgt * v.y;
        acc.z += wgt * v.z;
        acc.w += wgt * v.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    reinterpret_cast<float4 *>(o + (b * HH + h) * (int64_t)DD)[threadIdx.x] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

static cudaError_t launch_tc(const AttnArgs &x, int nsplit, float *out_rows, float *part_ml, cudaStream_t stream)
{
    TcArgs a;
    a.q = x.q;
    a.kv_rot = x.win;
    a.C = x.C;
    a.c8 = x.c8;
    a.c8_scale = x.c8_scale;
    a.c_rope = x.c_rope;
    a.idx = x.idx;
    a.sinks = x.sinks;
    a.part_ml = part_ml;
    a.status = x.status;
    a.S = x.R;
    a.T = x.T;
    a.P = x.P;
    a.k = x.idx != nullptr ? x.k : 0;
    a.W = x.W;
    a.m = x.m;
    a.decode = x.decode;
    a.nsplit = nsplit;
    a.scale_log2 = x.scale * 1.4426950408889634f;
    a.log2_theta_tok = x.log2_theta_tok;
    a.log2_theta_cmp = x.log2_theta_cmp;
    const size_t smem = 1024 + OFF_LIST + sizeof(int) * (size_t)std::max(a.k, 1);
    CUtensorMap tq;
    if (!make_tmap_bf16_sw128(&tq, x.q, (uint64_t)x.R * HH, DD, 64)) return cudaErrorInvalidValue;
    a.o = out_rows;   // final rows, or the split partials
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attend_tc_kernel<<<(unsigned)(x.R * nsplit), NUM_THREADS, smem, stream>>>(tq, a);
    return cudaGetLastError();
}

cudaError_t launch_attend_tc(const AttnArgs &x, cudaStream_t stream)
{
    if (x.R == 0) return cudaSuccess;
    return launch_tc(x, 1, x.o, nullptr, stream);
}

size_t attend_tc_decode_partials(int64_t B, int nsplit)
{
    return nsplit <= 1 ? 0 : (size_t)B * nsplit * HH * (DD + 2) * sizeof(float);
}

// Decode: nsplit CTAs per sequence write partials into `part` (attend_tc_decode_partials bytes),
// then one combine launch produces o. nsplit == 1 writes o directly.
cudaError_t launch_attend_tc_decode(const AttnArgs &x, int nsplit, float *part, cudaStream_t stream)
{
    if (x.R == 0) return cudaSuccess;
    if (nsplit <= 1) return launch_tc(x, 1, x.o, nullptr, stream);
    float *part_o = part;
    float *part_ml = part + (size_t)x.R * nsplit * HH * DD;
    cudaError_t e = launch_tc(x, nsplit, part_o, part_ml, stream);
    if (e != cudaSuccess) return e;
    combine_splits_kernel<<<(unsigned)(x.R * HH), 128, 0, stream>>>(part_o, part_ml, x.sinks, nsplit, x.o);
    return cudaGetLastError();
}

}  // namespace csa
