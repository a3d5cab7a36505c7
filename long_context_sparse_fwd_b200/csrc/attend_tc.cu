// attend_tc.cu -- CSA / HCA attention on the 5th-generation tensor cores (H=64, D=512, rope 64):
// a persistent kernel, one CTA per SM walking the queries (prefill rows, or decode sequence splits).
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
// are brought 64 at a time by TMA into 128-byte-swizzled shared memory (window rows as 2-D tiles,
// entries by four-row gathers), where the same tile is the K-major B operand of S = Q K^T and the
// MN-major B operand of O += P V: the selected rows are read from L2/HBM once and shared by all
// 64 heads. Three key stages.
// Q lives in TMEM as the A operand of S, so shared memory holds only keys and P, and the S
// MMA reads only the key tile from shared memory.
//   TMEM (M=64 uses 16 lanes of each 32-lane quarter, "half 0" = lanes +0..15, "half 1" = +16..31):
//     half 0: S_b   cols [0,64), [64,128)   double-buffered logits (on the lanes of Q, as the
//                                  A-from-TMEM MMA requires)
//             Q     cols [128,512) a ring of 12 chunk slots (32 columns each: 64 dims as bf16
//                                  pairs); query n puts its chunk c (the rope chunk rotated
//                                  with theta_cmp) in slot (8n + c) mod 12, so the next query's
//                                  chunks 0-3 are written while the current one still computes
//     half 1: O     cols [0,512)   output dims 0..511
// The two branches rotate their rope slices with different thetas. Once a window block has
// landed, the planner turns the rope slice of each window key by t * (f_cmp - f_tok) per pair
// (f = theta^(-2p/64)): a window key then scores against the theta_cmp-rotated q exactly as it
// did against the theta_tok-rotated one (rotations preserve dot products), and its value, rotated
// back by -t * f_cmp at the end, comes out rotated by -t * f_tok as required. So one rope chunk
// of q, one rope accumulator and one rotation back serve both branches.
// Softmax runs in the exp2 domain with a reference max per head that is only raised when a block
// exceeds it by more than 2^8 (then O is rescaled in TMEM after the previous P V completes),
// so almost every block needs no rescale. The sink seeds the reference and the running sum.
// TMEM is read and written with the 16-lane x2 access shape, so both halves of a warp work on the
// 16 heads of its quarter (each thread one head, half of the columns).
// Roles: warps 0-3 softmax + epilogue; warps 4-7 load keys (each warp a quarter of the block's
// rows, TMA issued by one elected lane; FP8 decode entries are converted by the whole warp) and
// write each query's Q into their TMEM quarter; warp 8 owns TMEM and issues MMAs from an event loop (a P V never waits for the next
// block's keys); warp 9 plans: it builds the next query's entry list, block range and rope table
// in a second slot and prefetches its Q into L2. Key blocks are counted over all of a CTA's
// queries, so the loaders run into the next query while the current one finishes; the next
// query's Q is written as soon as the last S of the current one has completed, and its first
// P V waits only until the epilogue has read O out of TMEM.
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
constexpr int NSTAGE = 3;                       // key stages
constexpr int KCHUNK = KB * 128;                // 8 KB
constexpr int STAGE = NCH * KCHUNK;             // 64 KB
constexpr int PBUF = HH * 128;                  // 8 KB
constexpr int NUM_THREADS = 320;
constexpr int SM_THREADS = 128;
constexpr int LOAD_WARP0 = 4;                   // warps 4..7 load keys and write Q
constexpr int LOAD_THREADS = 128;
constexpr int MMA_WARP = 8;
constexpr int PLAN_WARP = 9;
constexpr int PLAN_CONSUMERS = 4 + 1 + 4;       // loader warps, MMA warp (one arrival), softmax warps
constexpr float TAU = 8.f;
constexpr uint32_t LANE16 = 16u << 16;
constexpr uint32_t COL_S = 0, COL_Q = 128;   // half 0
constexpr int QSLOTS = 12;                   // Q chunk slots (32 columns each) from COL_Q

// TMEM slot of chunk c of the CTA's n-th query: consecutive queries share no slot of their first
// four chunks with the query before, so those are written before that query's last S completes.
__device__ __forceinline__ uint32_t q_slot(int64_t n, int c) { return (uint32_t)((8 * (int)(n % 3) + c) % QSLOTS); }
constexpr uint32_t COL_O2 = 256;             // half 1: O dims 256..511 (dims 0..255 at column 0)
constexpr int ROPE_TAB = 3 * 32 * 2;         // floats per slot: [tok, cmp, cmp - tok][pair][cos, sin]
constexpr uint32_t TMEM_COLS = 512;

constexpr size_t OFF_KV = 0;
constexpr size_t OFF_P = OFF_KV + (size_t)NSTAGE * STAGE;     // 192 KB
constexpr size_t OFF_ROPE = OFF_P + 2 * (size_t)PBUF;         // 208 KB: rope tables [2 slots][ROPE_TAB]
constexpr size_t OFF_PLAN = OFF_ROPE + 2 * ROPE_TAB * 4;
constexpr size_t OFF_BAR = OFF_PLAN + 128;
constexpr size_t OFF_LIST = OFF_BAR + 256;                    // entry lists [2 slots][k rounded up to 4]

struct TcArgs {
    const uint16_t *q;        // [R, 64, 512] (R = S prefill rows or B decode sequences)
    const uint16_t *kv_rot;   // prefill: [S, 512] window rows; decode: [B, W, 512] (positions P-W+1..P)
    const uint16_t *C;        // prefill: [T, 512]; decode: [B, T, 512] bf16 (or null: FP8 cache)
    const uint8_t *c8;        // decode FP8 cache: [B, T, 448] E4M3 codes
    const float *c8_scale;    //                   [B, T]
    const uint16_t *c_rope;   //                   [B, T, 64] bf16
    const int32_t *idx;       // [R, k] or null (HCA: every visible entry)
    const float *sinks;       // [64]
    float *o;                 // [R, 64, 512] (or split partials [R*nsplit, 64, 512])
    float *part_ml;           // split partials: [R*nsplit, 64, 2] (log2-domain reference max, sum)
    int32_t *status;
    int64_t S, T, P;          // S: prefill rows; P: decode position
    int64_t pos0;             // prefill: position of row 0 (window rows indexed by position)
    int k, W, m, decode, nsplit;
    float scale_log2;         // softmax scale * log2(e)
    double log2_theta_tok, log2_theta_cmp;
};

// What the planner hands to the other roles for one query (double-buffered with its entry list
// and rope table).
struct Plan {
    int64_t row;       // prefill query row, or decode sequence
    int64_t win_row;   // kv_rot row holding the first window key
    int32_t nw, ne;    // window keys, selected (valid) entries
    int32_t nbw;       // window blocks of the whole key list
    int32_t gb0, nb;   // this unit's key blocks: [gb0, gb0 + nb) of (window blocks, entry blocks)
    int32_t split;
    int32_t pad[2];
};
static_assert(sizeof(Plan) == 48, "plan layout");
static_assert(2 * sizeof(Plan) <= 128, "plan slots");

__device__ __forceinline__ uint4 ldg_hint(const uint4 *p, uint64_t policy)
{
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

// Registers written by a tcgen05.ld are read only after tcgen05.wait::ld: this empty asm, placed
// after the wait, keeps the compiler from moving their uses above it.
__device__ __forceinline__ void reg_fence(float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i) asm volatile("" : "+f"(v[i]));
}

// Wait (at most 100 ms) for a phase regardless of the abort flag: used before exit so that no
// copy or MMA is still writing this CTA's shared memory or TMEM.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 100000000ull) return;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// byte offset of 16-byte unit `u` (0..7) of row `row` inside a 128-byte-swizzled [rows x 128 B] chunk
__device__ __forceinline__ uint32_t sw128(int row, int u) { return (uint32_t)(row * 128 + ((u ^ (row & 7)) << 4)); }

// Rotate the 16 bf16 pairs in w (interleaved RoPE pairs p0 .. p0+15) by the angles of table `cs`
// ([pair][cos, sin]); result packed as bf16 pairs.
__device__ __forceinline__ void rotate16(const uint32_t (&w)[16], const float *cs, int p0, uint32_t (&out)[16])
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float x0 = bf_lo(w[i]), x1 = bf_hi(w[i]);
        const float c = cs[(p0 + i) * 2], s = cs[(p0 + i) * 2 + 1];
        out[i] = pack_bf2(x0 * c - x1 * s, x0 * s + x1 * c);
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                 const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o, TcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sKV = smem + OFF_KV;
    uint8_t *sP = smem + OFF_P;
    float *rope_tab = reinterpret_cast<float *>(smem + OFF_ROPE);   // [slot][tok, cmp, cmp - tok][pair][cos, sin]
    Plan *plans = reinterpret_cast<Plan *>(smem + OFF_PLAN);         // [slot]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    // A stage's loads complete on kv_full (entry blocks) or kv_wfull (window blocks): each barrier
    // then counts the uses of one kind in order, so every waiter waits exactly one phase ahead.
    uint64_t *kv_full = bars + 0;      // [stage] loader arrivals, entry blocks
    uint64_t *kv_empty = bars + 3;     // [stage] MMA commit
    uint64_t *s_full = bars + 6;       // [2] MMA commit
    uint64_t *p_ready = bars + 8;      // [2] 128 softmax arrivals
    // P V completion: block g (counted over all of this CTA's queries) commits o_done[g & 1]. When
    // the softmax of block g waits for P V of block g-1, the previous completion of that barrier
    // (block g-3) is already known to be done (it preceded S of block g), so a parity wait cannot
    // mistake an older phase for the one wanted.
    uint64_t *o_done = bars + 10;      // [2]
    uint64_t *o_final = bars + 12;     // [query & 1] every MMA of the query has completed
    uint64_t *o_free = bars + 14;      // 128 epilogue arrivals: O of the query has been read from TMEM
    uint64_t *q_free = bars + 15;      // MMA commit after the last S of a query
    uint64_t *q_ready = bars + 16;     // 128 loader arrivals: Q of the query is in TMEM
    uint64_t *plan_ready = bars + 17;  // [slot] planner
    uint64_t *plan_free = bars + 19;   // [slot] 4 loader warps + MMA + 4 softmax warps
    uint64_t *drain = bars + 21;       // single use: every MMA issued has completed
    uint64_t *kv_rdy = bars + 22;      // [stage] planner: a window block's rope slice has been turned
    uint64_t *kv_wfull = bars + 25;    // [stage] loader arrivals, window blocks
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 28);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 29);
    uint64_t *tab_ready = bars + 30;   // single use: the first query's rope tables are written
    int *elist_all = reinterpret_cast<int *>(smem + OFF_LIST);    // [slot][kcap]
    const int kcap = (max(a.k, 1) + 3) & ~3;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool partial = a.nsplit > 1;
    const int64_t units = a.S * a.nsplit;   // prefill: one query row each; decode: (sequence, split)

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&kv_full[i], 4);   // one arrival (expect_tx, or after FP8 stores) per loader warp
            mbar_init(&kv_empty[i], 1);
            mbar_init(&kv_rdy[i], 1);
            mbar_init(&kv_wfull[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_ready[i], SM_THREADS);
            mbar_init(&o_done[i], 1);
            mbar_init(&o_final[i], 1);
            mbar_init(&plan_ready[i], 1);
            mbar_init(&plan_free[i], PLAN_CONSUMERS);
        }
        mbar_init(o_free, SM_THREADS);
        mbar_init(q_free, 1);
        mbar_init(q_ready, LOAD_THREADS);
        mbar_init(drain, 1);
        mbar_init(tab_ready, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_ptr, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    // Launched as a programmatic dependent (decode), this grid may start before the top-k kernel
    // that writes the index lists has finished: only the planner waits for it, right before it
    // reads the first list, so the rope tables and the first query's Q load overlap that kernel.
    grid_launch_dependents();

    if (warp == PLAN_WARP) {
        // ====== planner: index list, block split and rope tables of each query; window rope turn ======
        int g = 0;           // key blocks of this CTA's earlier queries
        uint32_t wpar = 0;   // per stage: parity of the next kv_wfull completion
        bool dep_waited = false;
        for (int64_t n = 0;; ++n) {
            const int64_t u = blockIdx.x + n * gridDim.x;
            if (u >= units) break;
            const int s = (int)(n & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&plan_free[s], (uint32_t)((n >> 1) & 1) ^ 1u, abort, a.status)))
                break;
            // prefill: rows longest-first over the grid; decode: nsplit units per sequence
            const int64_t row = a.decode ? u / a.nsplit : a.S - 1 - u;
            const int split = a.decode ? (int)(u % a.nsplit) : 0;
            if (lane == 0 && (!a.decode || split == 0))   // bring this query's Q into L2 ahead of its use
                for (int dc = 0; dc < NCH; ++dc) tma_prefetch_2d(&tm_q, dc * 64, (int)(row * HH));
            const int64_t t = a.decode ? a.P : a.pos0 + row;          // position of the query
            const int64_t vis = a.decode ? a.T : visible_entries(t, a.m, a.T);
            const int64_t wpos0 = max((int64_t)0, t - a.W + 1);
            const int nw = (int)(t - wpos0 + 1);
            {   // rope tables: angle t * f_p (f_p = theta^(-2p/64)) for both thetas, and their difference
                float *rt = rope_tab + s * ROPE_TAB;
                float c, sn;
                rope_cos_sin((double)t, lane, RR, a.log2_theta_tok, &c, &sn);
                rt[lane * 2] = c;
                rt[lane * 2 + 1] = sn;
                rope_cos_sin((double)t, lane, RR, a.log2_theta_cmp, &c, &sn);
                rt[64 + lane * 2] = c;
                rt[64 + lane * 2 + 1] = sn;
                const double e = -(2.0 * lane / (double)RR);
                const double dang = (double)t * (exp2(e * a.log2_theta_cmp) - exp2(e * a.log2_theta_tok));
                double sd, cd;
                sincos(dang, &sd, &cd);
                rt[128 + lane * 2] = (float)cd;
                rt[128 + lane * 2 + 1] = (float)sd;
            }
            if (n == 0) {   // the loaders write this query's Q into TMEM as soon as its tables exist
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(tab_ready);
                grid_dependency_wait();   // the index lists
                dep_waited = true;
            }
            int *elist = elist_all + s * kcap;
            int ne;
            if (a.idx != nullptr) {   // compacted entry list (CSA); HCA uses entries 0..vis-1 directly
                const int32_t *ir = a.idx + row * (int64_t)a.k;
                int vals[32];   // k <= 1024: all loads in flight at once
#pragma unroll
                for (int i = 0; i < 32; ++i) vals[i] = i * 32 + lane < a.k ? __ldg(ir + i * 32 + lane) : -1;
                int cnt = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = vals[i];
                    const bool valid = e >= 0 && (int64_t)e < vis;
                    if (e >= 0 && !valid) report(a.status, CSA_ERR_INVALID_ARG);
                    const unsigned mk = __ballot_sync(0xffffffffu, valid);
                    if (valid) elist[cnt + __popc(mk & ((1u << lane) - 1u))] = e;
                    cnt += __popc(mk);
                }
                ne = cnt;
            } else {
                ne = (int)vis;
            }
            if (lane == 0) {
                const int nbw = (nw + KB - 1) / KB, nb_all = nbw + (ne + KB - 1) / KB;
                Plan p;
                p.row = row;
                p.win_row = a.decode ? row * a.W + (a.W - nw) : wpos0;
                p.nw = nw;
                p.ne = ne;
                p.nbw = nbw;
                // this unit's share of the key blocks (window blocks first, then the entry blocks)
                p.gb0 = (int)((int64_t)split * nb_all / a.nsplit);
                p.nb = (int)((int64_t)(split + 1) * nb_all / a.nsplit) - p.gb0;
                p.split = split;
                plans[s] = p;
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) mbar_arrive(&plan_ready[s]);

            const Plan pl = plans[s];
            // Turn the rope slice of this unit's window keys (see the header) once each window
            // block has landed; the MMA waits for kv_rdy on window blocks.
            // lane l always turns 16-byte unit (l & 7) of a key row: pairs 4(l & 7) .. +3
            float tc4[4], ts4[4];
            {
                const float *dt = rope_tab + s * ROPE_TAB + 128;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    tc4[e] = dt[((lane & 7) * 4 + e) * 2];
                    ts4[e] = dt[((lane & 7) * 4 + e) * 2 + 1];
                }
            }
            bool ok = true;
            for (int b = 0; b < pl.nb && pl.gb0 + b < pl.nbw; ++b) {
                const int gg = g + b, st = gg % NSTAGE;
                if (!__all_sync(0xffffffffu, mbar_wait(&kv_wfull[st], (wpar >> st) & 1u, abort, a.status))) {
                    ok = false;
                    break;
                }
                wpar ^= 1u << st;
                uint8_t *rope_rows = sKV + st * STAGE + (NCH - 1) * KCHUNK;   // dims 448..511 of each key
                uint4 v[16];   // all 16 of this lane's units (rows 4j + lane/8) loaded before any is turned
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    v[j] = *reinterpret_cast<const uint4 *>(rope_rows + sw128(j * 4 + (lane >> 3), lane & 7));
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                    uint32_t o4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = bf_lo(w4[e]), x1 = bf_hi(w4[e]);
                        o4[e] = pack_bf2(x0 * tc4[e] - x1 * ts4[e], x0 * ts4[e] + x1 * tc4[e]);
                    }
                    *reinterpret_cast<uint4 *>(rope_rows + sw128(j * 4 + (lane >> 3), lane & 7)) =
                        make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&kv_rdy[st]);
            }
            if (!ok) break;
            g += pl.nb;
        }
        if (!dep_waited) grid_dependency_wait();   // never finish before the kernel this one depends on
    } else if (warp < 4) {
        // =============== softmax + epilogue (warp w owns TMEM quarter w: heads 16w..16w+15) ===============
        const int hl = lane & 15, hf = lane >> 4;   // head of this thread, which half of the columns
        const int h = warp * 16 + hl;
        const uint32_t tq0 = tmem + ((uint32_t)(warp * 32) << 16);   // half 0 of the quarter
        const uint32_t tq1 = tq0 + LANE16;                            // half 1
        // the sink seeds the running max and sum; split partials leave it to the combine step
        const float zl = partial ? -INFINITY : a.sinks[h] * 1.4426950408889634f;
        if (threadIdx.x == 0) prefetch_tmap(&tm_o);
        int g = 0;   // key blocks of this CTA's earlier queries
        bool ok = true;
        for (int64_t n = 0;; ++n) {
            const int64_t u = blockIdx.x + n * gridDim.x;
            if (u >= units) break;
            const int s = (int)(n & 1);
            ok = __all_sync(0xffffffffu, mbar_wait(&plan_ready[s], (uint32_t)((n >> 1) & 1), abort, a.status));
            if (!ok) break;
            const Plan pl = plans[s];
            const float *rope_cmp = rope_tab + s * ROPE_TAB + 64;
            const int nb = pl.nb, gb0 = pl.gb0, nbw = pl.nbw;
            float m_ref = zl, l = (zl == -INFINITY) ? 0.f : 1.f;
            for (int b = 0; b < nb && ok; ++b) {
                const int gg = g + b;
                const int buf = gg & 1;
                const int gb = gb0 + b;
                const int nk = gb < nbw ? min(KB, pl.nw - gb * KB) : min(KB, pl.ne - (gb - nbw) * KB);
                ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (uint32_t)((gg >> 1) & 1), abort, a.status));
                if (!ok) break;
                tc_fence_after();
                float sv[32];   // logits of keys 32*hf .. 32*hf+31 for head h
                tmem_ld_half32(tq0 + COL_S + (uint32_t)buf * 64, sv);
                tmem_wait_ld();
                float mb = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    sv[j] = hf * 32 + j < nk ? sv[j] * a.scale_log2 : -INFINITY;
                    mb = fmaxf(mb, sv[j]);
                }
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));   // the partner thread holds the same head
                float corr = 1.f;
                bool need = false;
                if (mb > m_ref + TAU) {
                    corr = exp2f(m_ref - mb);
                    m_ref = mb;
                    l *= corr;
                    need = b > 0;
                }
                float sum = 0.f;
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const uint32_t w = pack_bf2(exp2f(sv[j] - m_ref), exp2f(sv[j + 1] - m_ref));
                    pk[j >> 1] = w;
                    sum += bf_lo(w) + bf_hi(w);
                }
                l += sum + __shfl_xor_sync(0xffffffffu, sum, 16);
                uint8_t *prow = sP + buf * PBUF;
#pragma unroll
                for (int uu = 0; uu < 4; ++uu)
                    *reinterpret_cast<uint4 *>(prow + sw128(h, hf * 4 + uu)) =
                        make_uint4(pk[uu * 4], pk[uu * 4 + 1], pk[uu * 4 + 2], pk[uu * 4 + 3]);
                if (__any_sync(0xffffffffu, need)) {
                    // O must hold every earlier P V of this query before it is rescaled
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&o_done[(gg - 1) & 1], (uint32_t)(((gg - 1) >> 1) & 1), abort, a.status));
                    tc_fence_after();
                    if (ok) {
#pragma unroll 1
                        for (uint32_t c = 0; c < DD; c += 64) {   // O (half 1)
                            const uint32_t ta = tq1 + c;
                            float v[32];
                            tmem_ld_half32(ta, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] *= corr;
                            tmem_st_half32(ta, v);
                        }
                        tmem_wait_st();
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&p_ready[buf]);
            }
            // ---------------- epilogue ----------------
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_final[s], (uint32_t)((n >> 1) & 1), abort, a.status));
            if (!ok) break;
            tc_fence_after();
            const int64_t orow = partial ? pl.row * a.nsplit + pl.split : pl.row;   // o holds partial rows
            float *orp = a.o + (orow * HH + h) * (int64_t)DD;
            if (nb > 0) {
                const float inv = partial ? 1.f : (l > 0.f ? 1.f / l : 0.f);
                // Each 64-column piece goes through this warp's own rows of the two P buffers
                // (32 rows of 128 B: row 16*hf + hl holds head 16w+hl, dims c + 32hf .. +31) and
                // leaves as whole 128-byte row segments, 8 lanes per segment.
                uint8_t *stage0 = sP + warp * 2048, *stage1 = sP + PBUF + warp * 2048;
                uint8_t *mine = (hf ? stage1 : stage0) + hl * 128;
                // Each staged piece leaves as two TMA tensor stores ([16 heads x 32 dims] each) issued by
                // lane 0, which also waits for the engine to have read the staging before it is reused.
                const int orow0 = (int)(orow * HH + warp * 16);
                auto emit = [&](float (&v)[32], int c) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] *= inv;
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
#pragma unroll
                    for (int uq = 0; uq < 8; ++uq)
                        *reinterpret_cast<float4 *>(mine + ((uq ^ (hl & 7)) << 4)) =
                            make_float4(v[4 * uq], v[4 * uq + 1], v[4 * uq + 2], v[4 * uq + 3]);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_o, stage0, c, orow0);
                        tma_store_2d(&tm_o, stage1, c + 32, orow0);
                        bulk_commit();
                    }
                };
                // The TMEM load of the next piece is in flight while the current one is written out.
                float va[32], vb[32];
                tmem_ld_half32(tq1, va);
#pragma unroll 1
                for (int c = 0; c < DD; c += 128) {
                    tmem_wait_ld();
                    reg_fence(va);
                    tmem_ld_half32(tq1 + (uint32_t)(c + 64), vb);
                    emit(va, c);
                    tmem_wait_ld();
                    reg_fence(vb);
                    if (c + 128 < DD) {
                        tmem_ld_half32(tq1 + (uint32_t)(c + 128), va);
                    } else {
                        tc_fence_before();
                        mbar_arrive(o_free);   // O has been read: the next query's P V may overwrite it
                        // rope dims 448..511: rotated back by -t * f_cmp (window keys were turned to match)
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const int p = hf * 16 + (j >> 1);
                            const float cc = rope_cmp[p * 2], sc = rope_cmp[p * 2 + 1];
                            const float e0 = vb[j], e1 = vb[j + 1];
                            vb[j] = e0 * cc + e1 * sc;
                            vb[j + 1] = -e0 * sc + e1 * cc;
                        }
                    }
                    emit(vb, c + 64);
                }
                if (lane == 0) bulk_wait_read_all();   // the P buffers are written again by the next query
                __syncwarp();
            } else {
                tc_fence_before();
                mbar_arrive(o_free);
                if (!partial) {
                    float4 *dst = reinterpret_cast<float4 *>(orp + hf * 256);
                    for (int i = 0; i < 64; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (partial && hf == 0) {   // reference max (log2 domain) and sum of this split; an empty split has l = 0
                float *ml = a.part_ml + (orow * HH + h) * 2;
                ml[0] = nb > 0 ? m_ref : -INFINITY;
                ml[1] = nb > 0 ? l : 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&plan_free[s]);
            g += nb;
        }
        if (lane == 0) bulk_wait_all();   // every output store of this warp has completed
        __syncwarp();
    } else if (warp >= LOAD_WARP0 && warp < MMA_WARP) {
        // ===== key loads (TMA into the swizzled stages) and Q into TMEM quarter lw =====
        const int lw = warp - LOAD_WARP0;        // key rows 16*lw .. 16*lw+15 of each block; heads 16*lw..
        const int hl = lane & 15, hf = lane >> 4;
        const uint32_t tqq = tmem + ((uint32_t)(lw * 32) << 16) + COL_Q;   // Q chunks, half 0 of quarter lw
        const uint64_t pol_once = policy_evict_first();   // q is read once
        // per stage (bit st): a load of each kind (window / entry) was issued, and the parity of the
        // phase the last one completes; used to drain the last loads before exit
        uint32_t w_issued = 0, w_par = 0, e_issued = 0, e_par = 0;
        if (lane == 0) {
            prefetch_tmap(&tm_c);
            prefetch_tmap(&tm_w);
        }
        // Q of the CTA's query qn into TMEM: thread (hl, hf) writes head 16*lw+hl, dims 64c + 32hf .. +31
        // of each chunk c. Chunks 0-3 go to slots that no S in flight reads (the query before last
        // has completed, which the previous call awaited), so they are written at once; chunks 4-7,
        // whose slots held chunks 0-3 of the previous query, once `ready` (every S of the previous
        // query has completed; for the first query, the rope tables exist) has completed.
        auto load_q = [&](int64_t qn, int64_t row, const float *rope_cs, uint64_t *ready, uint32_t ready_par) -> bool {
            const uint4 *qsrc = reinterpret_cast<const uint4 *>(a.q + (row * HH + lw * 16 + hl) * (int64_t)DD + hf * 32);
            uint4 x[16];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = ldg_hint(qsrc + half * 32 + (i >> 2) * 8 + (i & 3), pol_once);
                if (half == 1) {
                    if (!__all_sync(0xffffffffu, mbar_wait(ready, ready_par, abort, a.status))) return false;
                    tc_fence_after();
                }
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int c = half * 4 + cc;
                    const uint32_t wq[16] = {x[4 * cc].x,     x[4 * cc].y,     x[4 * cc].z,     x[4 * cc].w,
                                             x[4 * cc + 1].x, x[4 * cc + 1].y, x[4 * cc + 1].z, x[4 * cc + 1].w,
                                             x[4 * cc + 2].x, x[4 * cc + 2].y, x[4 * cc + 2].z, x[4 * cc + 2].w,
                                             x[4 * cc + 3].x, x[4 * cc + 3].y, x[4 * cc + 3].z, x[4 * cc + 3].w};
                    const uint32_t ta = tqq + q_slot(qn, c) * 32;
                    if (c < NCH - 1) {
                        tmem_st_half16u(ta, wq);
                    } else {   // rope dims: rotated with theta_cmp
                        uint32_t r[16];
                        rotate16(wq, rope_cs + 64, hf * 16, r);
                        tmem_st_half16u(ta, r);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(q_ready);
            return true;
        };
        // The first query's Q needs no plan: it is written as soon as the planner's rope tables exist
        // (before the index lists are awaited), while its first keys are being planned.
        bool run = true;
        if ((int64_t)blockIdx.x < units) {
            const int64_t u0 = blockIdx.x;
            run = load_q(0, a.decode ? u0 / a.nsplit : a.S - 1 - u0, rope_tab, tab_ready, 0u);
        }
        int g = 0;
        for (int64_t n = 0; run; ++n) {
            const int64_t u = blockIdx.x + n * gridDim.x;
            if (u >= units) break;
            const int s = (int)(n & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&plan_ready[s], (uint32_t)((n >> 1) & 1), abort, a.status))) break;
            const Plan pl = plans[s];
            const int *elist = elist_all + s * kcap;
            const float *rope_cs = rope_tab + s * ROPE_TAB;
            const int64_t ent_row0 = a.decode ? pl.row * a.T : 0;   // row of entry 0 in the entry tensor map
            bool ok = true;
            for (int b = 0; b <= pl.nb; ++b) {
                if (n > 0 && b == min(1, pl.nb)) {
                    // Q of this query, once every S of the previous query has completed
                    if (!load_q(n, pl.row, rope_cs, q_free, (uint32_t)((n - 1) & 1))) {
                        ok = false;
                        break;
                    }
                }
                if (b == pl.nb) break;
                const int gg = g + b;
                const int st = gg % NSTAGE, gb = pl.gb0 + b;
                if (!__all_sync(0xffffffffu, mbar_wait(&kv_empty[st], (uint32_t)((gg / NSTAGE) & 1) ^ 1u, abort, a.status))) {
                    ok = false;
                    break;
                }
                const bool win = gb < pl.nbw;
                const int kbase = win ? gb * KB : (gb - pl.nbw) * KB;
                const int nk = win ? min(KB, pl.nw - kbase) : min(KB, pl.ne - kbase);
                if (!win && a.C == nullptr) {
                    // FP8 entry cache: codes * per-entry scale on channels [0,448), bf16 rope on [448,512),
                    // converted to bf16 here and stored into the swizzled stage. Lane j < 28 handles
                    // channels [16j, 16j+16) of each row, lanes 28..31 the rope channels 448 + 16*(lane-28).
                    // The loads of 8 rows are issued together before any is converted.
                    uint8_t *stage = sKV + st * STAGE;
                    const int d0 = lane < 28 ? 16 * lane : 448 + 16 * (lane - 28);
                    const int dc = d0 >> 6, u0 = (d0 & 63) >> 3;
                    int my_e = 0;   // entry (row of the flattened cache) of key 16*lw + lane, lanes < 16
                    if (lane < 16) {
                        const int kk = kbase + min(lw * 16 + lane, nk - 1);
                        my_e = (int)(pl.row * a.T + (a.idx != nullptr ? elist[kk] : kk));
                    }
#pragma unroll 1
                    for (int r0 = 0; r0 < 16; r0 += 8) {
                        uint4 raw[8], rope1[8];
                        float sc[8];
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            const int64_t e = __shfl_sync(0xffffffffu, my_e, r0 + r);
                            if (lane < 28) {
                                sc[r] = __ldg(a.c8_scale + e);
                                raw[r] = __ldg(reinterpret_cast<const uint4 *>(a.c8 + e * 448) + lane);
                            } else {
                                const uint4 *rr = reinterpret_cast<const uint4 *>(a.c_rope + e * 64);
                                raw[r] = __ldg(rr + 2 * (lane - 28));
                                rope1[r] = __ldg(rr + 2 * (lane - 28) + 1);
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            const int key = lw * 16 + r0 + r;
                            uint4 o0, o1;
                            if (key >= nk) {   // padding keys hold zeros
                                o0 = make_uint4(0u, 0u, 0u, 0u);
                                o1 = o0;
                            } else if (lane < 28) {
                                const uint32_t cw[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
                                uint32_t ow[8];
#pragma unroll
                                for (int q2 = 0; q2 < 8; ++q2) {
                                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                                        (__nv_fp8x2_storage_t)((cw[q2 >> 1] >> ((q2 & 1) * 16)) & 0xffffu), __NV_E4M3);
                                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
                                    ow[q2] = pack_bf2(f.x * sc[r], f.y * sc[r]);
                                }
                                o0 = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                                o1 = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                            } else {
                                o0 = raw[r];
                                o1 = rope1[r];
                            }
                            *reinterpret_cast<uint4 *>(stage + dc * KCHUNK + sw128(key, u0)) = o0;
                            *reinterpret_cast<uint4 *>(stage + dc * KCHUNK + sw128(key, u0 + 1)) = o1;
                        }
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&kv_full[st]);
                    continue;
                }
                // Loader warp lw fills key rows 16*lw .. 16*lw+15 of the stage, 16 KB, with one elected lane
                // issuing: a window block is consecutive kv_rot rows (a [16 x 64] tile per 64-dim chunk);
                // a selected-entry block is a gather (four rows per gather4, per chunk), an all-entries block
                // (HCA) consecutive tiles. Every slot receives a real row: window and HCA slots past the last
                // key read the rows that follow (or the zero fill past the tensor), selected-entry slots past
                // the last key repeat it, so masked keys always hold finite values.
                uint8_t *stage = sKV + st * STAGE + lw * 16 * 128;
                uint64_t *bar = win ? &kv_wfull[st] : &kv_full[st];
                if (win) {
                    const int y = (int)(pl.win_row + kbase + lw * 16);
                    if (elect_one()) {
                        mbar_arrive_expect_tx(bar, 16 * 1024);
#pragma unroll
                        for (int dc = 0; dc < NCH; ++dc) tma_load_2d(stage + dc * KCHUNK, &tm_w, bar, dc * 64, y);
                    }
                    w_par = (w_issued >> st) & 1u ? w_par ^ (1u << st) : w_par;
                    w_issued |= 1u << st;
                } else if (a.idx == nullptr) {
                    // every visible entry (HCA): the block's rows are consecutive, one [16 x 64] tile per
                    // chunk as for the window; rows past the last key are later entries or the zero fill
                    const int y = (int)(ent_row0 + kbase + lw * 16);
                    if (elect_one()) {
                        mbar_arrive_expect_tx(bar, 16 * 1024);
#pragma unroll
                        for (int dc = 0; dc < NCH; ++dc) tma_load_2d(stage + dc * KCHUNK, &tm_c, bar, dc * 64, y);
                    }
                    e_par = (e_issued >> st) & 1u ? e_par ^ (1u << st) : e_par;
                    e_issued |= 1u << st;
                } else {
                    int my_row = 0;
                    if (lane < 16) {
                        const int kk = kbase + min(lw * 16 + lane, nk - 1);
                        my_row = (int)(ent_row0 + elist[kk]);
                    }
                    int r4[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) r4[i] = __shfl_sync(0xffffffffu, my_row, i);
                    if (elect_one()) {
                        mbar_arrive_expect_tx(bar, 16 * 1024);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                            for (int dc = 0; dc < NCH; ++dc)
                                tma_gather4(stage + dc * KCHUNK + q4 * 512, &tm_c, bar, dc * 64, r4[4 * q4], r4[4 * q4 + 1],
                                            r4[4 * q4 + 2], r4[4 * q4 + 3]);
                    }
                    e_par = (e_issued >> st) & 1u ? e_par ^ (1u << st) : e_par;
                    e_issued |= 1u << st;
                }
                __syncwarp();
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&plan_free[s]);
            g += pl.nb;
        }
        // never leave with copies in flight into this CTA's shared memory (after an abort some loads
        // may not have been consumed): wait, bounded, for the last load of each kind into each stage
        for (int i = 0; i < NSTAGE; ++i) {
            if ((w_issued >> i) & 1u) mbar_drain(&kv_wfull[i], (w_par >> i) & 1u);
            if ((e_issued >> i) & 1u) mbar_drain(&kv_full[i], (e_par >> i) & 1u);
        }
    } else if (warp == MMA_WARP) {
        // =============== MMA issuer: event loop per query ===============
        // The whole warp runs the loop (every decision is made warp-uniform with a vote) and one
        // elected lane issues the MMAs and commits: with warp-uniform control flow the descriptors
        // stay in uniform registers and each tcgen05.mma issues without per-instruction overhead.
        // The loop polls with test_wait: a failing try_wait may park the warp until that barrier
        // completes, which would hold back an S whose keys are ready behind a softmax still running.
        const uint32_t idS = idesc_bf16(64, 64);
        const uint32_t idPV = idesc_bf16(64, 256, true);
        // descriptors are formed once; a tile / k-step offset is added to the start-address field
        const uint64_t dK = sdesc_sw128(smem_u32(sKV), 16, 1024);
        const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);
        const uint64_t dV = sdesc_sw128(smem_u32(sKV), KCHUNK, 1024);
        int g = 0;
        uint32_t wpar = 0;   // per stage: parity of the next kv_rdy completion (window blocks)
        uint32_t epar = 0;   // per stage: parity of the next kv_full completion (entry blocks)
        for (int64_t n = 0;; ++n) {
            const int64_t u = blockIdx.x + n * gridDim.x;
            if (u >= units) break;
            const int s = (int)(n & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&plan_ready[s], (uint32_t)((n >> 1) & 1), abort, a.status))) break;
            const int nb = plans[s].nb, gb0 = plans[s].gb0, nbw = plans[s].nbw;
            if (!__all_sync(0xffffffffu, mbar_wait(q_ready, (uint32_t)(n & 1), abort, a.status))) break;
            tc_fence_after();
            int nS = 0, nPV = 0;
            bool ofree = n == 0;      // O of the previous query has been read out
            bool ok = true;
            // The timeout clock is read only while the loop is idle (every 256 polls without
            // progress): a read of the global timer is slow and would delay the next issue.
            uint64_t t_idle = 0;
            uint32_t polls = 0;
            while (nPV < nb) {
                bool progressed = false;
                // S(nS) needs its keys and a free logits buffer (softmax of nS-2 finished, i.e. PV(nS-2) issued)
                const int gs = g + nS;
                const int sst = gs % NSTAGE;
                const bool swin = gb0 + nS < nbw;   // window block: wait until its rope slice is turned
                if (nS < nb && nS <= nPV + 1 &&
                    __all_sync(0xffffffffu, swin ? mbar_test_wait(&kv_rdy[sst], (wpar >> sst) & 1u)
                                                 : mbar_test_wait(&kv_full[sst], (epar >> sst) & 1u))) {
                    if (swin) wpar ^= 1u << sst;
                    else epar ^= 1u << sst;
                    fence_async_smem();   // keys were written by cp.async (generic proxy); the MMA reads via the async proxy
                    tc_fence_after();
                    if (elect_one()) {
                        const uint32_t d = tmem + COL_S + (uint32_t)(gs & 1) * 64;
#pragma unroll
                        for (int dc = 0; dc < NCH; ++dc) {
                            const uint32_t qa = tmem + COL_Q + q_slot(n, dc) * 32;
                            const uint64_t kb = dK + ((sst * STAGE + dc * KCHUNK) >> 4);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) mma_bf16_ts(d, qa + ks * 8, kb + 2 * ks, idS, (dc | ks) != 0);
                        }
                        mma_commit(&s_full[gs & 1]);
                        if (nS + 1 == nb) mma_commit(q_free);
                    }
                    __syncwarp();
                    ++nS;
                    progressed = true;
                }
                if (!ofree && nPV < nS) ofree = __all_sync(0xffffffffu, mbar_test_wait(o_free, (uint32_t)((n - 1) & 1)));
                // PV(nPV) needs the softmax of block nPV (and, for the first, O of the previous query read out)
                const int gp = g + nPV;
                if (ofree && nPV < nS && __all_sync(0xffffffffu, mbar_test_wait(&p_ready[gp & 1], (uint32_t)((gp >> 1) & 1)))) {
                    tc_fence_after();
                    const int b = nPV, st = gp % NSTAGE;
                    if (elect_one()) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad = dP + (((gp & 1) * PBUF + ks * 32) >> 4);
                            const uint64_t vb = dV + ((st * STAGE + ks * 2048) >> 4);
                            mma_bf16(tmem + LANE16, ad, vb, idPV, b > 0 || ks > 0);                                 // dims 0..255
                            mma_bf16(tmem + LANE16 + COL_O2, ad, vb + ((4 * KCHUNK) >> 4), idPV, b > 0 || ks > 0);   // 256..511
                        }
                        mma_commit(&kv_empty[st]);
                        mma_commit(&o_done[gp & 1]);
                        if (b + 1 == nb) mma_commit(&o_final[s]);
                    }
                    __syncwarp();
                    ++nPV;
                    progressed = true;
                }
                if (progressed) {
                    polls = 0;
                } else if ((++polls & 255u) == 0) {
                    if (__any_sync(0xffffffffu, *abort != 0)) { ok = false; break; }
                    const uint64_t now = __shfl_sync(0xffffffffu, globaltimer(), 0);
                    if (polls == 256u) t_idle = now;   // first idle check since the last progress
                    if (now - t_idle > 2000000000ull) {
                        if (lane == 0) {
                            *abort = 1;
                            report(a.status, CSA_ERR_TIMEOUT);
                        }
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) break;
            if (elect_one()) {
                if (nb == 0) {   // nothing to compute: release Q and complete the query's phases
                    mma_commit(q_free);
                    mma_commit(&o_final[s]);
                }
                mbar_arrive(&plan_free[s]);
            }
            __syncwarp();
            g += nb;
        }
        // leave only when every MMA and commit issued has completed
        if (elect_one()) mma_commit(drain);
        __syncwarp();
        mbar_drain(drain, 0);
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
constexpr int COMBINE_MAX = 16;   // the most splits a decode call uses (HCA decode)

// NMAX: the most splits this instance takes (its registers hold one row of each).
template <int NMAX>
__global__ void __launch_bounds__(128)
combine_splits_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml, const float *__restrict__ sinks,
                      int nsplit, float *__restrict__ o)
{
    const int64_t b = blockIdx.x / HH;
    const int h = blockIdx.x % HH;
    const float z = sinks[h] * 1.4426950408889634f;
    grid_dependency_wait();   // the split partials
    // Every split's (max, sum) and partial row are loaded at once (at most NMAX splits). An empty split's
    // row was never written: it is left out by a select, so whatever the memory holds never reaches the sum.
    float mi[NMAX], li[NMAX];
    float4 v[NMAX];
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
        if (i < nsplit) {
            const int64_t r = (b * nsplit + i) * HH + h;
            mi[i] = part_ml[r * 2];
            li[i] = part_ml[r * 2 + 1];
            v[i] = reinterpret_cast<const float4 *>(part_o + r * (int64_t)DD)[threadIdx.x];
        }
    }
    float M = z;
#pragma unroll
    for (int i = 0; i < NMAX; ++i)
        if (i < nsplit) M = fmaxf(M, mi[i]);
    float L = (z == -INFINITY) ? 0.f : exp2f(z - M);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
        if (i < nsplit && mi[i] != -INFINITY && li[i] != 0.f) {
            const float wgt = exp2f(mi[i] - M);
            L += wgt * li[i];
            acc.x += wgt * v[i].x;
            acc.y += wgt * v[i].y;
            acc.z += wgt * v[i].z;
            acc.w += wgt * v[i].w;
        }
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
    a.pos0 = x.decode ? 0 : x.pos0;
    a.k = x.idx != nullptr ? x.k : 0;
    a.W = x.W;
    a.m = x.m;
    a.decode = x.decode;
    a.nsplit = nsplit;
    a.scale_log2 = x.scale * 1.4426950408889634f;
    a.log2_theta_tok = x.log2_theta_tok;
    a.log2_theta_cmp = x.log2_theta_cmp;
    const size_t smem = 1024 + OFF_LIST + 2 * sizeof(int) * (size_t)((std::max(a.k, 1) + 3) & ~3);
    CUtensorMap tq, tc, tw;
    if (!make_tmap_bf16_sw128(&tq, x.q, (uint64_t)x.R * HH, DD, 64)) return cudaErrorInvalidValue;
    // entry rows (gather4: one-row boxes) and window rows (16-row tiles); row coordinates are int32
    const uint64_t c_rows = x.decode ? (uint64_t)x.R * x.T : (uint64_t)x.T;
    const uint64_t w_rows = x.decode ? (uint64_t)x.R * x.W : (uint64_t)(x.pos0 + x.R);
    if (c_rows >= (1ull << 31) || w_rows >= (1ull << 31)) return cudaErrorInvalidValue;
    if (x.C != nullptr && c_rows > 0) {
        // selected entries (CSA) are gathered four one-row boxes at a time; every visible entry (HCA)
        // is read as consecutive 16-row tiles
        if (!make_tmap_bf16_sw128(&tc, x.C, c_rows, DD, x.idx != nullptr ? 1 : 16)) return cudaErrorInvalidValue;
    } else {
        tc = tq;   // FP8 cache (converted by the loader warps) or no entries: never used
    }
    if (w_rows > 0) {
        if (!make_tmap_bf16_sw128(&tw, x.win, w_rows, DD, 16)) return cudaErrorInvalidValue;
    } else {
        tw = tq;   // no window rows: never used
    }
    a.o = out_rows;   // final rows, or the split partials
    CUtensorMap to;   // output rows [R * 64 (or R * nsplit * 64), 512] fp32, stored as [16 x 32] boxes
    const uint64_t o_rows = (uint64_t)x.R * (uint64_t)nsplit * HH;
    if (o_rows >= (1ull << 31) || !make_tmap_f32_sw128(&to, out_rows, o_rows, DD, 16)) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(attend_tc_kernel), smem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM walks the units (query rows, or sequence splits) with stride grid
    int dev = 0, sms = 0;
    if ((e = current_device_sms(&dev, &sms)) != cudaSuccess) return e;
    const int64_t units = x.R * nsplit;
    const unsigned grid = (unsigned)std::min<int64_t>(units, std::max(sms, 1));
    if (x.after_kernel)
        return launch_dependent(attend_tc_kernel, dim3(grid), dim3(NUM_THREADS), smem, stream, tq, tc, tw, to, a);
    attend_tc_kernel<<<grid, NUM_THREADS, smem, stream>>>(tq, tc, tw, to, a);
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
    if (nsplit > COMBINE_MAX) return cudaErrorInvalidValue;
    float *part_o = part;
    float *part_ml = part + (size_t)x.R * nsplit * HH * DD;
    cudaError_t e = launch_tc(x, nsplit, part_o, part_ml, stream);
    if (e != cudaSuccess) return e;
    auto combine = [&](auto kern) {
        return launch_dependent(kern, dim3((unsigned)(x.R * HH)), dim3(128), 0, stream, (const float *)part_o,
                                (const float *)part_ml, x.sinks, nsplit, x.o);
    };
    if (nsplit <= 2) return combine(combine_splits_kernel<2>);
    if (nsplit <= 4) return combine(combine_splits_kernel<4>);
    if (nsplit <= 8) return combine(combine_splits_kernel<8>);
    return combine(combine_splits_kernel<COMBINE_MAX>);
}

}  // namespace csa
