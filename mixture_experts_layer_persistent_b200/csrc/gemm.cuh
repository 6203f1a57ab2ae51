// gemm.cuh -- persistent, warp-specialised grouped GEMM on tcgen05/TMEM (sm_100a).
//
// One template serves every contraction of the layer.  A group is one expert
// (routed experts first, then shared experts) and owns a contiguous range of
// "sorted rows" (the expert-major order of (token, slot) pairs).
//
//   ragged-M (forward, data gradients):  D[rows of g, N] = A[rows of g, K] . B_g[N, K]^T
//   ragged-K (weight gradients):         D_g[M, N] = sum over rows r of g of A[r, M]^T B[r, N]
//   router (one group of all tokens, split over K): partial logits of x . [Wr_hi|Wr_mid|Wr_lo]^T
//
// Operand rows that belong to a token are pulled by index straight from the
// token matrix into the shared-memory ring by two pull warps issuing 16-byte
// cp.async copies (the pull-at-dispatch idea of "Cursor åpner
// megakernelen…", paragraph on pulling versus pushing tokens, re-derived for
// one GPU: the expert tile fetches its rows instead of a separate scatter
// pass).  The push epilogue writes each output row to its (token, slot) row
// (push at combine, same paragraph).  The shared-memory stage ring walks a
// fixed-size buffer at tile granularity whatever the routing imbalance (the
// fixed-size macrobatch ring of "Megakernels are dead and back…", section
// "Números de MoK").
//
// Roles: warp 0 issues TMA loads of the contiguous operands into a
// STAGES-deep ring, warp 1 allocates TMEM and issues tcgen05.mma (one elected
// thread), warps 2-5 drain the double-buffered TMEM accumulator and run the
// epilogue, staging each 32-row block through shared memory so that global
// stores cover whole lines, and warps 6-9 (kernels with a gathered operand)
// pull the gathered rows.  TMA gather4 would also serve, but at four 128-byte
// rows per instruction it issues too slowly to keep the tensor core fed.
// Every output tile is produced by exactly one CTA with a fixed K order, so
// results do not depend on scheduling: the layer is bit-reproducible.
#pragma once
#include "ptx.cuh"
#include "quant.cuh"

namespace mok {

constexpr int BM = 128;        // UMMA M (cta_group::1, all 128 TMEM lanes)
constexpr int BK = 64;         // one 128-byte swizzle row of bf16
constexpr int kMaxGroups = 264;
constexpr int kPanelM = 8;     // ragged-M raster panel height (M tiles)
// cp.async pull warps of a kernel with a gathered operand (or MXFP8 activation
// scales): two, so that with the TMA producer, the MMA issuer and the four
// epilogue warps a CTA is 8 warps, two per SM sub-partition, and a thread may
// hold up to 255 registers (10 warps put three on two sub-partitions: 168)
constexpr int kPullWarps = 2;

enum Epi : int { EPI_SWIGLU = 0, EPI_PUSH = 1, EPI_DSWIGLU = 2, EPI_WGRAD = 3, EPI_ROUTER = 4 };

constexpr int kGemmBarBytes = 256;                 // mbarriers, abort flag, schedule slots of one phase
constexpr int kGemmAuxBytes = 3 * kMaxGroups * 4;  // group offsets, tile starts, group order

struct GemmArgs {
    int num_groups;               // G
    int num_routed;               // groups [0, num_routed) use tmB, the rest tmB_s / out_s
    const int *offsets;           // [G+1] sorted-row range of every group
    const int *gorder;            // ragged-K: group processing order (longest first), [G]
    const int *row_token;         // [R] gather row of each sorted row
    const int *row_slot;          // [R] destination row of each sorted row (push)
    const float *row_w;           // [R] routing weight of each sorted row
    int n_tiles;                  // output tiles along N (router: K splits)
    int m_tiles;                  // ragged-K: output tiles along M
    int num_kb;                   // ragged-M: K / BK (router: K blocks per split)
    int b_rows_per_group;         // ragged-M: rows of one group in B's 2D view
    int b_half;                   // EPI_SWIGLU: row offset of the up projection inside a group
    int a_k_mod;                  // EPI_ROUTER: A's K coordinate wraps at this many elements (H)
    const __nv_bfloat16 *gather_src; // token matrix the pull warps gather rows from (x or dy)
    int gather_ld;                // elements per token row of gather_src
    // MXFP8 (block-scaled) operands: ue8m0 scales, one byte per 32 K-elements, rows of sf_ld bytes
    const uint8_t *sfa_src;       // scales of A's rows (token rows when A is gathered, sorted rows otherwise)
    const uint8_t *sfb_src;       // scales of the routed groups' B rows (packed weight-scale layout)
    const uint8_t *sfb_src_s;     // scales of the shared groups' B rows (packed weight-scale layout)
    int sf_ld;                    // A scale bytes per row (K / 32)
    int sfb_row_tiles;            // 128-row blocks of the routed weight tensor
    int sfb_row_tiles_s;          // 128-row blocks of the shared weight tensor
    uint8_t *out_scales;          // MXFP8 SwiGLU epilogue: scales of h [R, I/32]; MXFP8 SwiGLU-backward
                                  // epilogue: scales of dGU [R, 2I/32]
    uint8_t *out_q;               // MXFP8 SwiGLU-backward epilogue: e4m3 codes of dGU [R, 2I]
    __nv_bfloat16 *out_hb;        // MXFP8 SwiGLU epilogue, training: the dequantised h [R, I] (with out2, out3)
    __nv_bfloat16 *out;           // main output
    __nv_bfloat16 *out_s;         // EPI_WGRAD: output of the shared groups
    __nv_bfloat16 *out2;          // EPI_SWIGLU: saved gate/up pre-activations [R, 2I] (or null)
    __nv_bfloat16 *out3;          // EPI_SWIGLU: w * h [R, I] (or null)
    float *out_f32;               // EPI_ROUTER: partial logits [n_tiles, rows, 256]; EPI_PUSH: fp32 slot rows
    float *const *push_dst;       // EPI_PUSH across ranks (expert parallelism): slot rows of every rank (fp32, or
                                  // bf16 in the MXFP8 forward); row_slot is then (rank << 24) | slot row, every
                                  // row a plain store (null: off)
    const __nv_bfloat16 *aux;     // EPI_DSWIGLU: saved gate/up pre-activations [R, 2I]
    const __nv_bfloat16 *aux_h;   // EPI_DSWIGLU: saved h [R, I] (the down GEMM's A operand)
    float *gpart;                 // EPI_DSWIGLU: <dy W_down, h> of each routed row over each N tile [R_routed, n_tiles]
    int ldo;                      // elements per output row
    int inter;                    // I
    int rows_total;               // EPI_ROUTER: rows of one partial-logit slab (T)
    long long group_out_elems;    // EPI_WGRAD: elements of one group's output
    int *status;                  // device status word
    int test_drop_signal;         // fault injection: CTA 0 skips its first accumulator signal
    int k_split;                  // ragged-K: > 0 limits the streaming kernel to groups with more rows
                                  // (a prefix of gorder); the resident kernel takes the rest
    int m_per_unit;               // resident weight-gradient kernel: M tiles per work unit
    int *sched;                   // tile counter of this launch, zero before it (one per launch)
    // Per-M-tile readiness between two ragged-M GEMMs of one persistent launch (the
    // gate/up GEMM produces the rows the down GEMM reads).  One counter per 128-row M
    // tile whatever either GEMM's tile height: counter of the M tile (g, mt) =
    // ready[(128-row M tiles of the groups before g) + mt], zero before the producing phase.
    int *ready;                   // null: no readiness tracking
    int ready_role;               // kReadySignal: each epilogue warp adds 1 per tile once its stores
                                  // are complete; kReadyWait: the producer waits for ready_target
                                  // before it hands a tile to the other roles
    int ready_target;
    const int *mt_base;           // kReadyWaitGroup: [G + 1] first 128-row M tile of each group (the
                                  // group's counters are mt_base[g] .. mt_base[g+1]-1)
};

// kReadyWaitGroup: a weight-gradient phase waits, before it loads a group's rows,
// until every M tile of the group has reached ready_target
constexpr int kReadyNone = 0, kReadySignal = 1, kReadyWait = 2, kReadyWaitGroup = 3;

template <int BN_, bool A_MN_, bool B_MN_, bool A_GATHER_, bool B_GATHER_, bool RAGGED_K_, int EPI_,
          bool MX_ = false, bool PAIR_ = false>
struct GemmCfg {
    static constexpr int BN = BN_;
    // Pair tiles: 256 rows of a group per tile, as two 128-row halves with their own
    // accumulator (TMEM columns 0.. and BN..) that share each weight stage.  An
    // expert of 129-256 rows then streams its weight strip once, in one CTA, whose
    // tensor core has time to spare while it waits for HBM, instead of a second
    // CTA running a whole K loop for a few rows.  The two accumulators take all of
    // TMEM, so a tile's epilogue is not overlapped with the next tile's MMAs.
    static constexpr bool PAIR = PAIR_;
    static constexpr int TM = PAIR ? 2 * BM : BM;                // rows per tile
    static constexpr bool A_MN = A_MN_, B_MN = B_MN_, A_GATHER = A_GATHER_, B_GATHER = B_GATHER_;
    static constexpr bool RAGGED_K = RAGGED_K_;
    static constexpr int EPI = EPI_;
    static constexpr bool MX = MX_;                              // e4m3 operands with ue8m0 block scales
    static constexpr int ESIZE = MX ? 1 : 2;                     // operand bytes per element
    static constexpr int KB_ELEMS = 128 / ESIZE;                 // K elements per 128-byte block row
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int A_STAGE = (PAIR ? 2 : 1) * A_BYTES;     // A halves, then B, in a stage
    static constexpr int STAGE_BYTES = A_STAGE + B_BYTES;
    static constexpr int SF_BYTES = MX ? 512 + BN * 4 : 0;       // SFA (128 rows) + SFB (BN rows), 4 bytes each
    // Tuning (measured at the DeepSeek-V3 shape): the weight-streaming kernels
    // want a deep operand ring; BN = 128 and MXFP8 trade a stage for a second
    // epilogue staging buffer so that one block's store overlaps the next
    // block's conversion; the weight gradients keep a deep ring.
    // Kernels whose epilogue moves several blocks per warp and tile (weight
    // gradients at N = 256, the MXFP8 down GEMM's fp32 pushes) do better with a
    // second staging buffer in place of a fourth stage; the plain weight
    // streamers, the MXFP8 gate/up GEMM among them (one block per warp and
    // tile), keep four.
    static constexpr bool MX_SWIGLU = MX && EPI == EPI_SWIGLU;
    // single-accumulator (MXFP8) epilogues hand the accumulator back to the MMA warp
    // as soon as its last columns are in registers, before their conversion and stores
    static constexpr bool EARLY_RELEASE = MX;
    static constexpr bool HEAVY_EPI = BN == 256 && ((MX && !MX_SWIGLU) || RAGGED_K);
    static constexpr int STAGES = (HEAVY_EPI || PAIR) ? 3 : (BN == 256 ? 4 : (RAGGED_K ? 6 : 5));
    static constexpr int EPI_BUFS = (HEAVY_EPI || (!RAGGED_K && BN != 256)) ? 2 : 1;
    static constexpr int EPI_WARPS = 4;
    static constexpr int PULL_WARPS = (A_GATHER || B_GATHER || MX) ? kPullWarps : 0;   // cp.async warps
    static constexpr int PULL_WARP0 = 2 + EPI_WARPS;
    static constexpr int THREADS = 64 + 32 * (EPI_WARPS + PULL_WARPS);
    static constexpr int GATHER_BYTES = A_GATHER ? A_STAGE : (B_GATHER ? B_BYTES : 0);
    // MXFP8: the weight scales of a K block (two 512-byte tiles) come with B
    static constexpr int TMA_BYTES = STAGE_BYTES - GATHER_BYTES + (MX ? 1024 : 0);
    static constexpr int ACC_BUFS = (MX || PAIR) ? 1 : 2;        // MXFP8 needs TMEM columns for the scales
    static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;
    static constexpr int SF_TMEM_COL = 256;                      // SFA at 256..259, SFB at 260..
    static constexpr int EPI_STAGE_BYTES = EPI_WARPS * EPI_BUFS * 4096;   // 32 x 128-byte blocks per epilogue warp
    // the epilogue staging blocks follow the scale region and must stay 1024-byte
    // aligned (their 128-byte swizzle phase comes from the address)
    static constexpr int SF_REGION = (STAGES * SF_BYTES + 1023) / 1024 * 1024;
    // ring, scale blocks and staging: the part of shared memory a GEMM phase carves
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES + SF_REGION + EPI_STAGE_BYTES;
    // standalone kernel: ring, then the phase's barrier block, group tables and TMEM slot
    static constexpr int SMEM_BYTES = 1024 + RING_BYTES + kGemmBarBytes + kGemmAuxBytes + 16;
    static constexpr uint32_t IDESC = idesc_bf16(BM, BN, A_MN, B_MN);
    static_assert(!MX || (!A_MN && !B_MN && !RAGGED_K && BN == 256 &&
                          (EPI == EPI_SWIGLU || EPI == EPI_PUSH || EPI == EPI_DSWIGLU)),
                  "MXFP8 serves the K-major expert GEMMs: the forward's and the data gradients'");
    static_assert(BN == 128 || BN == 256, "BN");
    static_assert(!PAIR || (!MX && !RAGGED_K && !A_MN && BN == 256), "pair tiles: BF16 with a K-major A");
    static_assert(!RAGGED_K || (A_MN && B_MN), "weight gradients take both operands MN-major");
    static_assert(!RAGGED_K || (A_GATHER != B_GATHER), "one operand of a weight gradient is gathered");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((STAGES * STAGE_BYTES) % 1024 == 0, "stage ring keeps 1024-byte alignment");
};

struct Tile {
    int g;          // group
    int nt;         // N tile (router: K split)
    int m0;         // ragged-M: first sorted row; ragged-K: first M index
    int rows;       // ragged-M: valid rows in the tile
    int krow0;      // ragged-K: first sorted row of the group
    int krows;      // ragged-K: rows of the group
    int nkb;        // K blocks
};

// gorder lists groups by rows descending: the first `nbig` have more than k_split rows
// (k_split <= 0: every group)
__device__ __forceinline__ int count_big_groups(const int *off, const int *order, int G, int k_split)
{
    if (k_split <= 0) return G;
    int lo = 0, hi = G;                   // first position whose group has <= k_split rows
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int g = order[mid];
        if (off[g + 1] - off[g] > k_split) lo = mid + 1; else hi = mid;
    }
    return lo;
}

template <class C>
__device__ __forceinline__ Tile decode_tile(int tile, const GemmArgs &a, const int *s_off, const int *s_tstart,
                                            const int *s_gorder, int G)
{
    Tile t;
    if constexpr (C::RAGGED_K) {
        const int tpg = a.m_tiles * a.n_tiles;
        const int gi = tile / tpg, local = tile - gi * tpg;
        t.g = s_gorder[gi];
        const int mt = local / a.n_tiles;
        t.nt = local - mt * a.n_tiles;
        t.m0 = mt * BM;
        t.rows = BM;
        t.krow0 = s_off[t.g];
        t.krows = s_off[t.g + 1] - t.krow0;
        t.nkb = (t.krows + BK - 1) / BK;
    } else {
        int lo = 0, hi = G - 1;          // largest g with s_tstart[g] <= tile
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        t.g = lo;
        // Raster inside a group: panels of up to kPanelM M tiles; within a panel
        // the N tiles are outer and the M tiles inner, so the CTAs that run at
        // the same time share one weight strip (read from HBM once) while the
        // panel's activation rows stay in L2.
        const int local = tile - s_tstart[lo];
        const int mtiles = (s_off[lo + 1] - s_off[lo] + C::TM - 1) / C::TM;
        const int per_panel = kPanelM * a.n_tiles;
        const int pnl = local / per_panel, rem = local - pnl * per_panel;
        const int ps = min(kPanelM, mtiles - pnl * kPanelM);
        t.nt = rem / ps;
        const int mt = pnl * kPanelM + (rem - t.nt * ps);
        t.m0 = s_off[lo] + mt * C::TM;
        t.rows = min(C::TM, s_off[lo + 1] - t.m0);
        t.krow0 = 0;
        t.krows = 0;
        t.nkb = a.num_kb;
    }
    return t;
}

// silu(g) = g sigmoid(g) with the hardware exponential and reciprocal (CUDA's
// __expf and __fdividef intrinsics: a few ulp of fp32, far inside the layer's
// tolerances); for g < -88, __expf(-g) is inf and the quotient 0
__device__ __forceinline__ float sigmoid_f(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_f(g); }

template <int N>
__device__ __forceinline__ void pack_bf16(const float *v, uint32_t *p)
{
#pragma unroll
    for (int i = 0; i < N / 2; ++i) p[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
}

// ---- tile schedule ----------------------------------------------------------
// Tiles start in index order.  CTA b takes tile b first; afterwards its
// producer claims the next index from the launch's counter kClaimAhead K blocks
// before the last load of its current tile (so the atomic's latency hides
// behind those loads) and hands it to the other roles through a ring of
// shared-memory slots.  The tiles that share a weight strip
// (an expert's M tiles of one N strip, adjacent in the raster) therefore start
// within about a microsecond of each other and read the strip from HBM once,
// where a fixed stride of gridDim.x lets the CTAs drift apart over the waves.
// A tile's result does not depend on the CTA that computes it.
constexpr int kSchedSlots = 4;
constexpr int kClaimAhead = 8;     // K blocks before a tile's last load at which the next tile is claimed

struct Sched {
    uint64_t *full;     // [kSchedSlots] slot written (one producer arrival)
    uint64_t *empty;    // [kSchedSlots] slot read by every consuming warp
    int *slot;          // [kSchedSlots] tile indices
};

// producer lane 0: publish the tile of turn `it` (total = no more work)
__device__ __forceinline__ bool sched_put(const Sched &s, int it, int tile, volatile int *abort_flag, int *status)
{
    const int k = it % kSchedSlots;
    if (!mbar_wait(&s.empty[k], (static_cast<uint32_t>(it / kSchedSlots) & 1u) ^ 1u, abort_flag, status)) return false;
    s.slot[k] = tile;
    mbar_arrive(&s.full[k]);             // release: the slot is visible to the waiters
    return true;
}

// a consuming warp: the tile of turn `it` (total when the work is out or a wait gave up)
__device__ __forceinline__ int sched_take(const Sched &s, int it, int total, int lane, volatile int *abort_flag,
                                          int *status)
{
    const int k = it % kSchedSlots;
    int tile = total;
    if (lane == 0) {
        if (mbar_wait(&s.full[k], static_cast<uint32_t>(it / kSchedSlots) & 1u, abort_flag, status)) tile = s.slot[k];
        mbar_arrive(&s.empty[k]);
    }
    return __shfl_sync(0xffffffffu, tile, 0);
}

// ---- epilogue block I/O --------------------------------------------------
// A warp moves 32 rows x 128 bytes at a time through its 4 KB staging buffer,
// laid out like a 128-byte-swizzled TMA box (16-byte chunk c of row r at
// chunk c ^ (r & 7)), so the TMA store engine writes whole lines while the
// warp moves on; the stores stay in flight without occupying the warp.

// The staging buffers of a warp rotate: before a buffer is rewritten, the store
// issued from it `bufs` blocks earlier must have read it (the bufs - 1 later
// store groups, one per block, may still be reading theirs).
struct EpiStage {
    uint32_t *buf;      // bufs x 1024 words
    int bufs;           // 1 to 4
    int cur;            // buffer of the next block
    __device__ __forceinline__ uint32_t *next()
    {
        uint32_t *b = buf + (cur << 10);
        cur = cur + 1 == bufs ? 0 : cur + 1;
        return b;
    }
};

// wait until at most `pending` bulk store groups of this thread still read shared memory
__device__ __forceinline__ void bulk_wait_read(int pending)
{
    switch (pending) {
    case 0: asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); break;
    default: asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory"); break;
    }
}

__device__ __forceinline__ void stage_block(const EpiStage &es, uint32_t *stg, const uint32_t *p, int lane)
{
    if (lane == 0) bulk_wait_read(es.bufs - 1);     // the store that last used this buffer has read it
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4 *>(stg + lane * 32 + ((c ^ (lane & 7)) << 2)) =
            make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
    fence_proxy_async_smem();
    __syncwarp();
}

// 32 full rows to rows row0..row0+31 of a row-major tensor, starting at column col
__device__ __forceinline__ void store_block_tile(EpiStage &es, const uint32_t *p, int lane, const CUtensorMap *tm,
                                                 int col, int row0)
{
    uint32_t *stg = es.next();
    stage_block(es, stg, p, lane);
    if (lane == 0) {
        tma_store_2d(tm, stg, col, row0);
        bulk_commit();
    }
}

// 32 full rows, row `lane` to row dst_row (this lane's value), starting at column col
__device__ __forceinline__ void store_block_scatter(EpiStage &es, const uint32_t *p, int lane, const CUtensorMap *tm,
                                                    int col, int dst_row)
{
    uint32_t *stg = es.next();
    stage_block(es, stg, p, lane);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int r0 = __shfl_sync(0xffffffffu, dst_row, 4 * q + 0);
        const int r1 = __shfl_sync(0xffffffffu, dst_row, 4 * q + 1);
        const int r2 = __shfl_sync(0xffffffffu, dst_row, 4 * q + 2);
        const int r3 = __shfl_sync(0xffffffffu, dst_row, 4 * q + 3);
        if (lane == 0) tma_scatter4(tm, stg + q * 128, col, r0, r1, r2, r3);
    }
    if (lane == 0) bulk_commit();
}

// one lane's 128-byte row with plain stores (blocks that are only partly valid)
__device__ __forceinline__ void store_row_direct(void *dst, const uint32_t *p)
{
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < 8; ++c) d[c] = make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
}

// 64 bytes (32 bf16) of this lane's own row with plain 16-byte stores
__device__ __forceinline__ void store_row64(void *dst, const uint32_t *p)
{
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < 4; ++c) d[c] = make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
}

// One 1x32 MXFP8 block of this lane's row: 32 e4m3 codes at q, the ue8m0 byte at sc
__device__ __forceinline__ void mx_store_block(const float (&v)[32], uint8_t *q, uint8_t *sc)
{
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_exponent(amax);
    uint32_t w[8];
    mx_codes32(v, e, w);
    uint4 *d = reinterpret_cast<uint4 *>(q);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
    *sc = static_cast<uint8_t>(e + 127);
}

// 128 bytes of this lane's own row (null = zeros) straight into registers: the
// first 16-byte load brings the line into L1 and the other seven hit it
__device__ __forceinline__ void load_row_direct(uint32_t *p, const void *src)
{
    const uint4 *q = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = src ? __ldg(q + c) : make_uint4(0u, 0u, 0u, 0u);
        p[4 * c] = v.x; p[4 * c + 1] = v.y; p[4 * c + 2] = v.z; p[4 * c + 3] = v.w;
    }
}

// ---- readiness between the phases of one persistent launch --------------------
__device__ __forceinline__ void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Order this thread's generic-proxy accesses with its async-proxy (TMA) accesses of global memory.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Producer lane: wait until the M tile's counter reaches the target (bounded;
// gives up as mbar_wait does).  Loads the tile's rows only after this returns true.
__device__ __forceinline__ bool wait_ready(const int *ctr, int target, volatile int *abort, int *status)
{
    if (ld_acquire_gpu(ctr) >= target) {
        fence_proxy_async_global();
        return true;
    }
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (ld_acquire_gpu(ctr) >= target) {
            fence_proxy_async_global();
            return true;
        }
        if ((i & 63u) == 0u && (*abort || globaltimer() - t0 > kWaitLimitNs)) {
            *abort = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Epilogue warp: this warp's rows of the tile are in global memory (its TMA stores
// complete, its plain stores fenced); count it on the tile's readiness counter.
__device__ __forceinline__ void signal_ready(int *ctr, int lane)
{
    __syncwarp();
    if (lane == 0) {
        bulk_wait0();
        fence_proxy_async_global();
        __threadfence();
        red_release_gpu_add(ctr, 1);
    }
    __syncwarp();
}

// Producer warp: wait for every M tile of group g (bounded, as wait_ready).  The
// 32 lanes check 32 M tiles' counters at a time (one round trip for a group of up
// to 4096 rows); the warp barrier and a fence then order every lane's acquire
// before the loads lane 0 issues.  Callers check a group once per CTA: a CTA's
// tiles (work units) of one group are claimed one after another.
__device__ __forceinline__ bool wait_group_ready(const GemmArgs &a, int g, int lane, volatile int *abort,
                                                 int *status)
{
    const int m0 = a.mt_base[g], m1 = a.mt_base[g + 1];
    const uint64_t t0 = globaltimer();
    for (int base = m0; base < m1; base += 32) {
        const int mt = base + lane;
        for (uint32_t i = 0;; ++i) {
            const bool done = mt >= m1 || ld_acquire_gpu(a.ready + mt) >= a.ready_target;
            if (__all_sync(0xffffffffu, done)) break;
            if ((i & 63u) == 63u) {
                const bool give_up = lane == 0 && (*abort || globaltimer() - t0 > kWaitLimitNs);
                if (__any_sync(0xffffffffu, give_up)) {
                    if (lane == 0) {
                        *abort = 1;
                        atomicOr(status, kStatusTimeout);
                    }
                    return false;
                }
            }
        }
    }
    __syncwarp();
    __threadfence();
    fence_proxy_async_global();
    return true;
}

// One grouped-GEMM phase run by every thread of the CTA.
//   smem       1024-byte aligned: C::RING_BYTES of stage ring, scale blocks and staging
//   bar_block  kGemmBarBytes of barriers for this phase alone (not reused by another phase)
//   aux        kGemmAuxBytes of group tables
//   tmem_base  TMEM columns [0, C::TMEM_COLS) allocated by the caller
// Starts and ends with a CTA-wide barrier.  A standalone launch wraps one phase;
// the persistent forward runs several in one launch.
template <class C>
__device__ __forceinline__ void gemm_phase(uint8_t *smem, uint64_t *bar_block, int *aux, uint32_t tmem_base,
                                           const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmB_s,
                                           const CUtensorMap &tmO, const CUtensorMap &tmO2, const CUtensorMap &tmO3,
                                           const GemmArgs &args)
{
    uint8_t *tiles = smem;
    uint8_t *sf_tiles = tiles + C::STAGES * C::STAGE_BYTES;     // MXFP8 scale blocks, one per stage
    uint32_t *epi_stage = reinterpret_cast<uint32_t *>(sf_tiles + C::SF_REGION);
    uint64_t *full_bar = bar_block;
    uint64_t *empty_bar = full_bar + C::STAGES;
    uint64_t *accf = empty_bar + C::STAGES;
    uint64_t *acce = accf + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acce + 2);
    const Sched sch{acce + 3, acce + 3 + kSchedSlots, reinterpret_cast<int *>(acce + 3 + 2 * kSchedSlots)};
    uint64_t *drain_bar = acce + 3 + 2 * kSchedSlots + (4 * kSchedSlots + 7) / 8;   // MMA drain on abort
    static_assert(8 * (2 * C::STAGES + 6 + 2 * kSchedSlots) + 4 * kSchedSlots <= kGemmBarBytes, "barrier region");
    int *s_off = aux;
    int *s_tstart = s_off + kMaxGroups;
    int *s_gorder = s_tstart + kMaxGroups;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.num_groups;
    int *status = args.status;

    if (warp == 0) {
        for (int i = lane; i <= G; i += 32) s_off[i] = args.offsets[i];
        if constexpr (C::RAGGED_K) {
            for (int i = lane; i < G; i += 32) s_gorder[i] = args.gorder[i];
        }
        __syncwarp();
        if constexpr (!C::RAGGED_K) {
            // tile prefix over groups: ceil(rows / TM) * n_tiles tiles each, and the first
            // 128-row M tile of each group, which indexes the readiness counters whatever
            // the tile height (warp scans; the second goes where ragged-K GEMMs keep the
            // group order)
            int carry = 0, mcarry = 0;
            for (int base = 0; base < G; base += 32) {
                const int g = base + lane;
                int v = 0, mv = 0;
                if (g < G) {
                    v = ((s_off[g + 1] - s_off[g] + C::TM - 1) / C::TM) * args.n_tiles;
                    mv = (s_off[g + 1] - s_off[g] + BM - 1) / BM;
                }
                int incl = v, mincl = mv;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, d);
                    const int mo = __shfl_up_sync(0xffffffffu, mincl, d);
                    if (lane >= d) {
                        incl += o;
                        mincl += mo;
                    }
                }
                if (g < G) {
                    s_tstart[g] = carry + incl - v;
                    s_gorder[g] = mcarry + mincl - mv;
                }
                carry += __shfl_sync(0xffffffffu, incl, 31);
                mcarry += __shfl_sync(0xffffffffu, mincl, 31);
            }
            if (lane == 0) s_tstart[G] = carry;
        }
        if (lane == 0) {
            for (int s = 0; s < C::STAGES; ++s) {
                mbar_init(&full_bar[s], 1 + 32 * C::PULL_WARPS);
                mbar_init(&empty_bar[s], 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(&accf[b], 1);
                mbar_init(&acce[b], 32 * C::EPI_WARPS);
            }
            for (int i = 0; i < kSchedSlots; ++i) {
                mbar_init(&sch.full[i], 1);
                mbar_init(&sch.empty[i], 1 + C::EPI_WARPS + C::PULL_WARPS);
            }
            mbar_init(drain_bar, 1);
            *abort_flag = 0;
            fence_barrier_init();
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmB_s);
            tma_prefetch_desc(&tmO);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // data an earlier phase of the same launch wrote with plain stores is read here
    // by TMA and cp.async: order the two proxies (free in a standalone launch)
    fence_proxy_async_global();
    const int total = C::RAGGED_K ? count_big_groups(s_off, s_gorder, G, args.k_split) * args.m_tiles * args.n_tiles
                                  : s_tstart[G];

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        int fills = 0;                   // stages whose loads this producer issued
        int ready_g = -1;                // ragged K: last group found complete
        int tile = blockIdx.x;
        for (int it = 0;; ++it) {
            bool put = true;
            if constexpr (C::RAGGED_K) {
                if (args.ready_role == kReadyWaitGroup && tile < total) {
                    // the group's rows of the contiguous operand come from an earlier phase
                    const Tile t = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
                    if (t.g != ready_g) {
                        put = wait_group_ready(args, t.g, lane, abort_flag, status);
                        ready_g = t.g;
                    }
                    if (!put) tile = total;
                }
            } else {
                if (args.ready_role == kReadyWait && tile < total) {
                    // the rows this tile reads are produced by an earlier phase of the launch
                    const Tile t = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
                    // (s_gorder holds each group's first 128-row M tile here; a pair tile
                    // needs both of its M tiles)
                    const int mt = s_gorder[t.g] + (t.m0 - s_off[t.g]) / BM;
                    if (lane == 0) {
                        put = wait_ready(args.ready + mt, args.ready_target, abort_flag, status);
                        if (C::PAIR && put && t.rows > BM)
                            put = wait_ready(args.ready + mt + 1, args.ready_target, abort_flag, status);
                    }
                    put = __shfl_sync(0xffffffffu, put, 0);
                    if (!put) tile = total;          // publish "no more work" to the other roles
                }
            }
            bool put2 = true;
            if (lane == 0) put2 = sched_put(sch, it, tile, abort_flag, status);
            put = __shfl_sync(0xffffffffu, put2, 0) && put;
            if (!put || tile >= total) break;
            const Tile t = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
            const bool routed = t.g < args.num_routed;
            const CUtensorMap *mB = routed ? &tmB : &tmB_s;
            const int gl = routed ? t.g : t.g - args.num_routed;
            if constexpr (C::RAGGED_K) {
                // weight gradients (MN-major operands, two and four boxes per K block, a
                // few K blocks per tile): the lanes issue the boxes in parallel after
                // lane 0's wait, which measured faster here than lane 0 alone
                const int claim_kb = t.nkb > kClaimAhead ? t.nkb - kClaimAhead : 0;
                int next = 0;
                if (t.nkb == 0 && lane == 0) next = static_cast<int>(gridDim.x) + atomicAdd(args.sched, 1);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (kb == claim_kb && lane == 0) next = static_cast<int>(gridDim.x) + atomicAdd(args.sched, 1);
                    bool ok = true;
                    if (lane == 0) {
                        ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, status);
                        if (ok) mbar_arrive_expect_tx(&full_bar[stage], C::TMA_BYTES);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) goto producer_done;
                    uint8_t *sA = tiles + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_STAGE;
                    uint64_t *fb = &full_bar[stage];
                    const int kg = C::EPI == EPI_ROUTER ? t.nt * args.num_kb + kb : kb;   // global K block
                    constexpr int KE = C::KB_ELEMS;
                    // ---- A (gathered A rows come from the pull warps)
                    if constexpr (!C::A_GATHER && !C::A_MN) {
                        if (lane == 0) {
                            const int kc = C::EPI == EPI_ROUTER ? (kg * BK) % args.a_k_mod : kb * KE;
                            tma_load_2d(sA, &tmA, fb, kc, t.m0);
                        }
                    } else if constexpr (!C::A_GATHER && C::A_MN) {
                        if (lane < BM / 64) tma_load_2d(sA + lane * 8192, &tmA, fb, t.m0 + lane * 64, t.krow0 + kb * BK);
                    }
                    // ---- B
                    if constexpr (!C::B_MN) {
                        if (lane == 0) {
                            if constexpr (C::EPI == EPI_SWIGLU) {
                                const int row = gl * args.b_rows_per_group + t.nt * 128;
                                tma_load_2d(sB, mB, fb, kb * KE, row);
                                tma_load_2d(sB + 128 * 128, mB, fb, kb * KE, row + args.b_half);
                            } else if constexpr (C::EPI == EPI_ROUTER) {
                                tma_load_2d(sB, mB, fb, kg * BK, 0);
                            } else {
                                tma_load_2d(sB, mB, fb, kb * KE, gl * args.b_rows_per_group + t.nt * C::BN);
                            }
                        }
                    } else if constexpr (!C::B_GATHER && !C::RAGGED_K) {
                        if (lane < C::BN / 64)
                            tma_load_2d(sB + lane * 8192, mB, fb, t.nt * C::BN + lane * 64,
                                        gl * args.b_rows_per_group + kb * BK);
                    } else if constexpr (!C::B_GATHER && C::RAGGED_K) {
                        if (lane < C::BN / 64)
                            tma_load_2d(sB + lane * 8192, &tmB, fb, t.nt * C::BN + lane * 64, t.krow0 + kb * BK);
                    }
                    if constexpr (C::MX) {
                        // the weight scales of this K block: one packed 512-byte tile per 128 B rows
                        if (lane == 0) {
                            const uint8_t *sb = routed ? args.sfb_src : args.sfb_src_s;
                            const long long rt = routed ? args.sfb_row_tiles : args.sfb_row_tiles_s;
                            const int r0 = gl * args.b_rows_per_group + (C::EPI == EPI_SWIGLU ? t.nt * 128 : t.nt * C::BN);
                            const int r1 = C::EPI == EPI_SWIGLU ? r0 + args.b_half : r0 + 128;
                            uint8_t *sf = sf_tiles + stage * C::SF_BYTES;
                            bulk_load(sf + 512, sb + (static_cast<long long>(kb) * rt + (r0 >> 7)) * 512, 512, fb);
                            bulk_load(sf + 1024, sb + (static_cast<long long>(kb) * rt + (r1 >> 7)) * 512, 512, fb);
                        }
                    }
                    ++fills;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tile = __shfl_sync(0xffffffffu, next, 0);
            } else {
                // lane 0 alone runs the tile's K loop
                const bool pair2 = C::PAIR && t.rows > BM;           // a pair tile's second half holds rows
                const int claim_kb = t.nkb > kClaimAhead ? t.nkb - kClaimAhead : 0;
                int next = 0;
                bool ok = true;
                if (lane == 0) {
                    // the tile's K loop by lane 0 alone (no warp-wide step per K block)
                    if (t.nkb == 0) next = static_cast<int>(gridDim.x) + atomicAdd(args.sched, 1);
                    for (int kb = 0; kb < t.nkb; ++kb) {
                        if (kb == claim_kb) next = static_cast<int>(gridDim.x) + atomicAdd(args.sched, 1);
                        ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, status);
                        if (!ok) break;
                        // a pair tile whose second half holds no rows loads only the first A half
                        mbar_arrive_expect_tx(&full_bar[stage],
                                              C::TMA_BYTES - (C::PAIR && !C::A_GATHER && !pair2 ? C::A_BYTES : 0));
                        uint8_t *sA = tiles + stage * C::STAGE_BYTES;
                        uint8_t *sB = sA + C::A_STAGE;
                        uint64_t *fb = &full_bar[stage];
                        const int kg = C::EPI == EPI_ROUTER ? t.nt * args.num_kb + kb : kb;   // global K block
                        constexpr int KE = C::KB_ELEMS;
                        // ---- A (gathered A rows come from the pull warps)
                        if constexpr (!C::A_GATHER && !C::A_MN) {
                            const int kc = C::EPI == EPI_ROUTER ? (kg * BK) % args.a_k_mod : kb * KE;
                            tma_load_2d(sA, &tmA, fb, kc, t.m0);
                            if constexpr (C::PAIR) {
                                if (pair2) tma_load_2d(sA + C::A_BYTES, &tmA, fb, kc, t.m0 + BM);
                            }
                        } else if constexpr (!C::A_GATHER && C::A_MN) {
#pragma unroll
                            for (int c = 0; c < BM / 64; ++c)
                                tma_load_2d(sA + c * 8192, &tmA, fb, t.m0 + c * 64, t.krow0 + kb * BK);
                        }
                        // ---- B
                        if constexpr (!C::B_MN) {
                            if constexpr (C::EPI == EPI_SWIGLU) {
                                const int row = gl * args.b_rows_per_group + t.nt * 128;
                                tma_load_2d(sB, mB, fb, kb * KE, row);
                                tma_load_2d(sB + 128 * 128, mB, fb, kb * KE, row + args.b_half);
                            } else if constexpr (C::EPI == EPI_ROUTER) {
                                tma_load_2d(sB, mB, fb, kg * BK, 0);
                            } else {
                                tma_load_2d(sB, mB, fb, kb * KE, gl * args.b_rows_per_group + t.nt * C::BN);
                            }
                        } else if constexpr (!C::B_GATHER && !C::RAGGED_K) {
#pragma unroll
                            for (int c = 0; c < C::BN / 64; ++c)
                                tma_load_2d(sB + c * 8192, mB, fb, t.nt * C::BN + c * 64, gl * args.b_rows_per_group + kb * BK);
                        } else if constexpr (!C::B_GATHER && C::RAGGED_K) {
#pragma unroll
                            for (int c = 0; c < C::BN / 64; ++c)
                                tma_load_2d(sB + c * 8192, &tmB, fb, t.nt * C::BN + c * 64, t.krow0 + kb * BK);
                        }
                        if constexpr (C::MX) {
                            // the weight scales of this K block: one packed 512-byte tile per 128 B rows
                            const uint8_t *sb = routed ? args.sfb_src : args.sfb_src_s;
                            const long long rt = routed ? args.sfb_row_tiles : args.sfb_row_tiles_s;
                            const int r0 = gl * args.b_rows_per_group + (C::EPI == EPI_SWIGLU ? t.nt * 128 : t.nt * C::BN);
                            const int r1 = C::EPI == EPI_SWIGLU ? r0 + args.b_half : r0 + 128;
                            uint8_t *sf = sf_tiles + stage * C::SF_BYTES;
                            bulk_load(sf + 512, sb + (static_cast<long long>(kb) * rt + (r0 >> 7)) * 512, 512, fb);
                            bulk_load(sf + 1024, sb + (static_cast<long long>(kb) * rt + (r1 >> 7)) * 512, 512, fb);
                        }
                        ++fills;
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) goto producer_done;
                tile = __shfl_sync(0xffffffffu, next, 0);
            }
        }
    producer_done:
        if (lane == 0) {
            // the last STAGES fills: after an abort, let their loads land (bounded) before
            // the CTA releases its shared memory; otherwise wait until the MMA has released
            // them, so that no arrival on this phase's barriers is still in flight when the
            // phase ends (a later phase of the launch may reuse the memory)
            const bool aborted = *abort_flag != 0;
            int s2 = stage;
            uint32_t ph = phase;
            for (int i = 0; i < min(fills, C::STAGES); ++i) {
                if (--s2 < 0) {
                    s2 = C::STAGES - 1;
                    ph ^= 1u;
                }
                mbar_drain(aborted ? &full_bar[s2] : &empty_bar[s2], ph);
            }
        }
    } else if (warp >= C::PULL_WARP0) {
        // ------------------------------------------------------------ pull warps
        // Gathered operand: each 128-byte row is copied by index from the token
        // matrix with 16-byte cp.async into the 128-byte-swizzled layout the MMA
        // descriptors expect (16-byte chunk c of row r lands at chunk c ^ (r & 7)).
        if constexpr (C::PULL_WARPS > 0) {
            constexpr int NP = 32 * C::PULL_WARPS;      // pull threads
            constexpr int RS = NP / 8;                  // a thread's rows are RS apart
            const int p = threadIdx.x - 32 * C::PULL_WARP0;
            const int c16 = p & 7;
            const int r0 = p >> 3;                      // 0 .. RS-1
            const uint8_t *src = reinterpret_cast<const uint8_t *>(args.gather_src);
            const size_t ld = static_cast<size_t>(args.gather_ld) * C::ESIZE;   // bytes per token row
            int stage = 0;
            uint32_t phase = 0;
            for (int it = 0;; ++it) {
                const int tile = sched_take(sch, it, total, lane, abort_flag, status);
                if (tile >= total) break;
                const Tile t = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
                if constexpr (!C::RAGGED_K) {
                    // K-major A: the tile's TM rows, this thread's rows r0 + RS i (a pair
                    // tile's second half only when it holds rows: the MMA skips it otherwise)
                    int tok[C::TM / RS];
                    const int copy_rows = C::PAIR && t.rows > BM ? C::TM : BM;
                    if constexpr (C::A_GATHER) {
#pragma unroll
                        for (int i = 0; i < C::TM / RS; ++i) {
                            const int r = r0 + RS * i;
                            tok[i] = r < t.rows ? __ldg(args.row_token + t.m0 + r) : 0;
                        }
                    }
                    // MXFP8 scales of A: rows p + NP q (their token rows when A is gathered);
                    // the weight scales come with B from the producer
                    const uint8_t *sfa[BM / NP];
                    if constexpr (C::MX) {
#pragma unroll
                        for (int q = 0; q < BM / NP; ++q) {
                            const int m = p + NP * q;
                            const int ar = m < t.rows ? (C::A_GATHER ? __ldg(args.row_token + t.m0 + m) : t.m0 + m)
                                                      : (C::A_GATHER ? 0 : t.m0);
                            sfa[q] = args.sfa_src + (size_t)ar * args.sf_ld;
                        }
                    }
                    for (int kb = 0; kb < t.nkb; ++kb) {
                        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, status)) goto pull_done;
                        if constexpr (C::A_GATHER) {
                            uint8_t *dst = tiles + stage * C::STAGE_BYTES;
#pragma unroll
                            for (int i = 0; i < C::TM / RS; ++i) {
                                const int r = r0 + RS * i;
                                if (C::TM == BM || r < copy_rows)
                                    cp_async16(dst + r * 128 + ((c16 ^ (r & 7)) << 4), src + tok[i] * ld + kb * 128 + c16 * 16);
                            }
                        }
                        if constexpr (C::MX) {
                            // SF atom layout: the 4 scales of row m at byte 16 (m % 32) + 4 (m / 32) of its 128-row block
                            uint8_t *sf = sf_tiles + stage * C::SF_BYTES;
#pragma unroll
                            for (int q = 0; q < BM / NP; ++q) {
                                const int m = p + NP * q;
                                cp_async4(sf + 16 * (m & 31) + 4 * (m >> 5), sfa[q] + kb * 4);
                            }
                        }
                        cp_async_arrive_noinc(&full_bar[stage]);
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                } else {
                    // MN-major operand: 64 gathered K rows per block, this thread's rows r0 + RS i
                    constexpr int CH = (C::A_GATHER ? BM : C::BN) / 64;
                    constexpr int NR = BK / RS;                 // rows per thread and K block
                    constexpr int OFF = C::A_GATHER ? 0 : C::A_STAGE;
                    const int mn0 = C::A_GATHER ? t.m0 : t.nt * C::BN;
                    const int end = t.krow0 + t.krows;
                    // token rows of K blocks kb, kb+1, kb+2: fetched three blocks ahead so
                    // that the index loads never stall the copies
                    int tk0[NR], tk1[NR], tk2[NR];
#pragma unroll
                    for (int i = 0; i < NR; ++i) {
                        const int kr = t.krow0 + r0 + RS * i;
                        tk0[i] = kr < end ? __ldg(args.row_token + kr) : 0;
                        tk1[i] = kr + BK < end ? __ldg(args.row_token + kr + BK) : 0;
                        tk2[i] = kr + 2 * BK < end ? __ldg(args.row_token + kr + 2 * BK) : 0;
                    }
                    for (int kb = 0; kb < t.nkb; ++kb) {
                        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, status)) goto pull_done;
                        uint8_t *dst = tiles + stage * C::STAGE_BYTES + OFF;
#pragma unroll
                        for (int i = 0; i < NR; ++i) {
                            const int r = r0 + RS * i;
                            const uint8_t *row = src + tk0[i] * ld + mn0 * C::ESIZE + c16 * 16;
#pragma unroll
                            for (int j = 0; j < CH; ++j)
                                cp_async16(dst + j * 8192 + r * 128 + ((c16 ^ (r & 7)) << 4), row + j * 128);
                        }
                        cp_async_arrive_noinc(&full_bar[stage]);
#pragma unroll
                        for (int i = 0; i < NR; ++i) {
                            const int kr = t.krow0 + (kb + 3) * BK + r0 + RS * i;
                            tk0[i] = tk1[i];
                            tk1[i] = tk2[i];
                            tk2[i] = kr < end ? __ldg(args.row_token + kr) : 0;
                        }
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        pull_done:
            cp_async_wait_all();         // nothing of this thread still lands in shared memory
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Lane 0 alone runs a tile's K loop: the tensor core queues about one MMA
        // beyond the one it executes, so every cycle the issuer spends between two
        // K blocks (a warp shuffle and barrier per block cost about a fifth of the
        // MMA rate) is tensor-core idle time; the warp joins once per tile.  The
        // weight gradients keep the warp in the loop (their last K block's tail rows
        // are zeroed by the 32 lanes).
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        for (int it = 0;; ++it) {
            const int tile = sched_take(sch, it, total, lane, abort_flag, status);
            if (tile >= total) break;
            const Tile t = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&acce[acc], acc_phase ^ 1u, abort_flag, status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
            if constexpr (C::RAGGED_K) {
                // weight gradients (a few K blocks per tile, the last one ragged): the
                // warp walks the K loop together, which measured faster here
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (lane == 0) ok = mbar_wait(&full_bar[stage], phase, abort_flag, status);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t *sA = tiles + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_STAGE;
                    if constexpr (C::RAGGED_K) {
                        const int valid = t.krows - kb * BK;
                        if (valid < BK) {
                            // rows past the group's end: zero them in the contiguous operand
                            // (the gathered operand holds finite rows there)
                            uint8_t *base = C::A_GATHER ? sB : sA;
                            const int chunks = C::A_GATHER ? C::BN / 64 : BM / 64;
                            const int n16 = (BK - valid) * 8;
                            for (int c = 0; c < chunks; ++c) {
                                uint4 *p = reinterpret_cast<uint4 *>(base + c * 8192 + valid * 128);
                                for (int i = lane; i < n16; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        if constexpr (C::PULL_WARPS > 0) fence_proxy_async_smem();   // cp.async data -> tensor core
                        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
                        if constexpr (C::MX) {
                            // scales of this K block into TMEM (issued before, so ordered with, the MMAs)
                            const uint32_t sf0 = smem_u32(sf_tiles + stage * C::SF_BYTES);
                            const uint32_t tsfa = tmem_base + C::SF_TMEM_COL, tsfb = tsfa + 4;
                            tmem_cp_32x128b_x4(tsfa, smem_desc_plain(sf0));
#pragma unroll
                            for (int b = 0; b < C::BN / 128; ++b) tmem_cp_32x128b_x4(tsfb + 4 * b, smem_desc_plain(sf0 + 512 + 512 * b));
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint64_t ad = smem_desc_sw128(a0 + k * 32, 16, 1024);
                                const uint64_t bd = smem_desc_sw128(b0 + k * 32, 16, 1024);
                                const uint32_t j = static_cast<uint32_t>(k);
                                umma_mxf8(d_tmem, ad, bd, idesc_mxf8(BM, C::BN, j), tsfa | (j << 30), tsfb | (j << 30),
                                          (kb | k) != 0 ? 1u : 0u);
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < BK / 16; ++k) {
                                const uint64_t ad = C::A_MN ? smem_desc_sw128(a0 + k * 2048, 8192, 1024)
                                                            : smem_desc_sw128(a0 + k * 32, 16, 1024);
                                const uint64_t bd = C::B_MN ? smem_desc_sw128(b0 + k * 2048, 8192, 1024)
                                                            : smem_desc_sw128(b0 + k * 32, 16, 1024);
                                umma_bf16(d_tmem, ad, bd, C::IDESC, (kb | k) != 0 ? 1u : 0u);
                            }
                        }
                        umma_commit(&empty_bar[stage]);
                    }
                    __syncwarp();
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            } else {
                // issue K block kb from stage st (lane 0); every lane advances stage / phase
                // itself, so the warp needs no broadcast of them
                const bool pair2 = C::PAIR && t.rows > BM;          // a pair tile's second half holds rows
                auto issue_kb = [&](int kb, int st) {
                    uint8_t *sA = tiles + st * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_STAGE;
                    if constexpr (C::PULL_WARPS > 0) fence_proxy_async_smem();   // cp.async data -> tensor core
                    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
                    if constexpr (C::MX) {
                        // scales of this K block into TMEM (issued before, so ordered with, the MMAs)
                        const uint32_t sf0 = smem_u32(sf_tiles + st * C::SF_BYTES);
                        const uint32_t tsfa = tmem_base + C::SF_TMEM_COL, tsfb = tsfa + 4;
                        tmem_cp_32x128b_x4(tsfa, smem_desc_plain(sf0));
#pragma unroll
                        for (int b = 0; b < C::BN / 128; ++b) tmem_cp_32x128b_x4(tsfb + 4 * b, smem_desc_plain(sf0 + 512 + 512 * b));
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ad = smem_desc_sw128(a0 + k * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(b0 + k * 32, 16, 1024);
                            const uint32_t j = static_cast<uint32_t>(k);
                            umma_mxf8(d_tmem, ad, bd, idesc_mxf8(BM, C::BN, j), tsfa | (j << 30), tsfb | (j << 30),
                                      (kb | k) != 0 ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            const uint64_t ad = C::A_MN ? smem_desc_sw128(a0 + k * 2048, 8192, 1024)
                                                        : smem_desc_sw128(a0 + k * 32, 16, 1024);
                            const uint64_t bd = C::B_MN ? smem_desc_sw128(b0 + k * 2048, 8192, 1024)
                                                        : smem_desc_sw128(b0 + k * 32, 16, 1024);
                            umma_bf16(d_tmem, ad, bd, C::IDESC, (kb | k) != 0 ? 1u : 0u);
                        }
                        if constexpr (C::PAIR) {
                            if (pair2) {
                                // the second half's rows against the same weight block
                                const uint32_t a1 = a0 + C::A_BYTES;
#pragma unroll
                                for (int k = 0; k < BK / 16; ++k) {
                                    const uint64_t bd = C::B_MN ? smem_desc_sw128(b0 + k * 2048, 8192, 1024)
                                                                : smem_desc_sw128(b0 + k * 32, 16, 1024);
                                    umma_bf16(d_tmem + C::BN, smem_desc_sw128(a1 + k * 32, 16, 1024), bd, C::IDESC,
                                              (kb | k) != 0 ? 1u : 0u);
                                }
                            }
                        }
                    }
                    umma_commit(&empty_bar[st]);
                };
                if (lane == 0) {
                    int st = stage;
                    uint32_t ph = phase;
                    for (int kb = 0; kb < t.nkb; ++kb) {
                        ok = mbar_wait(&full_bar[st], ph, abort_flag, status);
                        if (!ok) break;
                        tc_fence_after();
                        issue_kb(kb, st);
                        if (++st == C::STAGES) {
                            st = 0;
                            ph ^= 1u;
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                for (int kb = 0; kb < t.nkb; ++kb)
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
            }
            if (lane == 0 && !(args.test_drop_signal && blockIdx.x == 0 && tile == 0)) {
                if (t.nkb > 0) umma_commit(&accf[acc]);
                else mbar_arrive(&accf[acc]);
            }
            __syncwarp();
            if (++acc == C::ACC_BUFS) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
            // the MMAs (and scale copies) this warp issued complete before TMEM is released
            if (lane == 0) {
                umma_commit(drain_bar);
                mbar_drain(drain_bar, 0);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int eq = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = eq * 32 + lane;          // tile row of this thread
        const int ew = warp - 2;                 // epilogue warp index
        EpiStage stg{reinterpret_cast<uint32_t *>(epi_stage) + ew * C::EPI_BUFS * 1024, C::EPI_BUFS, 0};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int it = 0;; ++it) {
            const int tile = sched_take(sch, it, total, lane, abort_flag, status);
            if (tile >= total) break;
            const Tile tt = decode_tile<C>(tile, args, s_off, s_tstart, s_gorder, G);
            if (!mbar_wait(&accf[acc], acc_phase, abort_flag, status)) break;
            tc_fence_after();
            // a pair tile's halves one after the other (accumulator columns 0.. and BN..)
            for (int hh = 0; hh < (C::PAIR ? 2 : 1); ++hh) {
                Tile t = tt;
                if constexpr (C::PAIR) {
                    t.m0 = tt.m0 + hh * BM;
                    t.rows = min(BM, tt.rows - hh * BM);
                    if (t.rows <= 0) break;
                }
                const uint32_t taddr = tmem_base + static_cast<uint32_t>((C::PAIR ? hh : acc) * C::BN) +
                                       (static_cast<uint32_t>(eq * 32) << 16);
                const bool valid = row < t.rows;
                const bool full = eq * 32 + 31 < t.rows;        // all 32 rows of this warp's block valid
                const int row0 = t.m0 + eq * 32;                // first row of the block (ragged-M)
                if constexpr (C::EPI == EPI_SWIGLU && C::MX) {
                    // h = silu(g) u quantised per 32 columns: e4m3 codes [R, I] and ue8m0 scales [R, I/32]
                    const int r = t.m0 + row;
                    const int I = args.inter;
                    const int n0 = t.nt * 128;
                    uint32_t q[32];
                    uint32_t sc = 0;
                    // the single accumulator is handed back to the MMA warp as soon as its
                    // last columns are in registers: the loads of block b + 1 overlap the
                    // math of block b
                    float gb[2][32], ub[2][32];
                    tmem_ld32(taddr, gb[0]);
                    tmem_ld32(taddr + 128, ub[0]);
                    tmem_ld_wait();
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        float *g = gb[blk & 1], *u = ub[blk & 1];
                        if (blk < 3) {
                            tmem_ld32(taddr + 32 * (blk + 1), gb[(blk + 1) & 1]);
                            tmem_ld32(taddr + 128 + 32 * (blk + 1), ub[(blk + 1) & 1]);
                        }
                        if (args.out2 && valid) {
                            // training: the gate and up pre-activations as bf16
                            uint32_t pg[16], pu[16];
                            pack_bf16<32>(g, pg);
                            pack_bf16<32>(u, pu);
                            store_row64(args.out2 + (size_t)r * 2 * I + n0 + 32 * blk, pg);
                            store_row64(args.out2 + (size_t)r * 2 * I + I + n0 + 32 * blk, pu);
                        }
                        float amax = 0.0f;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            g[i] = silu_f(g[i]) * u[i];
                            amax = fmaxf(amax, fabsf(g[i]));
                        }
                        const int e = mx_exponent(amax);
                        mx_codes32(g, e, q + 8 * blk);
                        sc |= static_cast<uint32_t>(e + 127) << (8 * blk);
                        if (args.out_hb && valid) {
                            // training: the dequantised h (exact in bf16) and w times it, rounded
                            const float w = args.row_w[r];
                            uint32_t ph[16], pw[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const uint32_t word = q[8 * blk + (i >> 1)] >> (16 * (i & 1));
                                const float h0 = mx_decode(word, e), h1 = mx_decode(word >> 8, e);
                                ph[i] = pack_bf16x2(h0, h1);
                                pw[i] = pack_bf16x2(w * h0, w * h1);
                            }
                            store_row64(args.out_hb + (size_t)r * I + n0 + 32 * blk, ph);
                            store_row64(args.out3 + (size_t)r * I + n0 + 32 * blk, pw);
                        }
                        if (blk < 3) tmem_ld_wait();
                        if (blk == 2) {
                            tc_fence_before();
                            mbar_arrive(&acce[acc]);         // every column of the accumulator is in registers
                        }
                    }
                    uint8_t *qout = reinterpret_cast<uint8_t *>(args.out);
                    if (full) store_block_tile(stg, q, lane, &tmO, n0, row0);
                    else if (valid) store_row_direct(qout + (size_t)r * I + n0, q);
                    if (valid) *reinterpret_cast<uint32_t *>(args.out_scales + (size_t)r * (I / 32) + t.nt * 4) = sc;
                } else if constexpr (C::EPI == EPI_SWIGLU) {
                    const int r = t.m0 + row;
                    const int I = args.inter;
                    const int n0 = t.nt * 128;
                    const float w = (valid && args.out3) ? args.row_w[r] : 0.0f;
#pragma unroll 1
                    for (int c = 0; c < 128; c += 64) {
                        uint32_t hp[32], wp[32];
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float g[32], u[32];
                            tmem_ld32(taddr + c + 32 * half, g);
                            tmem_ld32(taddr + 128 + c + 32 * half, u);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * u[i];
                            pack_bf16<32>(g, hp + 16 * half);
#pragma unroll
                            for (int i = 0; i < 32; ++i) g[i] = w * bf16_round(g[i]);
                            pack_bf16<32>(g, wp + 16 * half);
                        }
                        if (full) store_block_tile(stg, hp, lane, &tmO, n0 + c, row0);
                        else if (valid) store_row_direct(args.out + (size_t)r * I + n0 + c, hp);
                        if (args.out3) {
                            if (full) store_block_tile(stg, wp, lane, &tmO3, n0 + c, row0);
                            else if (valid) store_row_direct(args.out3 + (size_t)r * I + n0 + c, wp);
                        }
                        if (args.out2) {
#pragma unroll
                            for (int part = 0; part < 2; ++part) {       // gate, then up pre-activations
                                float v[64];
                                uint32_t p[32];
                                tmem_ld32(taddr + 128 * part + c, *reinterpret_cast<float(*)[32]>(v));
                                tmem_ld32(taddr + 128 * part + c + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                                tmem_ld_wait();
                                pack_bf16<64>(v, p);
                                const int col = part * I + n0 + c;
                                if (full) store_block_tile(stg, p, lane, &tmO2, col, row0);
                                else if (valid) store_row_direct(args.out2 + (size_t)r * 2 * I + col, p);
                            }
                        }
                    }
                } else if constexpr (C::EPI == EPI_PUSH && C::MX) {
                    const int dst_row = valid ? args.row_slot[t.m0 + row] : 0;
                    if (args.out_f32) {
                        // MXFP8 gate/up dgrad: fp32 rows pushed into their (token, slot) row; across
                        // ranks into the dX slot rows of the token's rank, with plain stores
                        float *fbase = args.out_f32;
                        int frow = dst_row;
                        if (args.push_dst) {
                            fbase = args.push_dst[dst_row >> 24];
                            frow = dst_row & ((1 << 24) - 1);
                        }
                        const bool ftma = full && !args.push_dst;
                        float *dst = fbase + (size_t)frow * args.ldo + t.nt * C::BN;
#pragma unroll 1
                        for (int c = 0; c < C::BN; c += 32) {
                            float v[32];
                            uint32_t p[32];
                            tmem_ld32(taddr + c, v);
                            tmem_ld_wait();
                            if (c == C::BN - 32) {
                                tc_fence_before();
                                mbar_arrive(&acce[acc]);         // every column of the accumulator is in registers
                            }
#pragma unroll
                            for (int i = 0; i < 32; ++i) p[i] = __float_as_uint(v[i]);
                            if (ftma) store_block_scatter(stg, p, lane, &tmO, t.nt * C::BN + c, dst_row);
                            else if (valid) store_row_direct(dst + c, p);
                        }
                    } else {
                        // MXFP8 forward: bf16 rows pushed into their (token, slot) row; across
                        // ranks into the slot rows of the token's rank, with plain stores
                        __nv_bfloat16 *obase = args.out;
                        int prow = dst_row;
                        if (args.push_dst) {
                            obase = reinterpret_cast<__nv_bfloat16 *>(args.push_dst[dst_row >> 24]);
                            prow = dst_row & ((1 << 24) - 1);
                        }
                        const bool tma = full && !args.push_dst;
                        __nv_bfloat16 *dst = obase + (size_t)prow * args.ldo + t.nt * C::BN;
#pragma unroll 1
                        for (int c = 0; c < C::BN; c += 64) {
                            float v[64];
                            uint32_t p[32];
                            tmem_ld32(taddr + c, *reinterpret_cast<float(*)[32]>(v));
                            tmem_ld32(taddr + c + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                            tmem_ld_wait();
                            if (c == C::BN - 64) {
                                tc_fence_before();
                                mbar_arrive(&acce[acc]);         // every column of the accumulator is in registers
                            }
                            pack_bf16<64>(v, p);
                            if (tma) store_block_scatter(stg, p, lane, &tmO, t.nt * C::BN + c, dst_row);
                            else if (valid) store_row_direct(dst + c, p);
                        }
                    }
                } else if constexpr (C::EPI == EPI_PUSH) {
                    // fp32 rows pushed into their (token, slot) row of the slot buffer; across
                    // ranks into the slot buffer of the token's rank, with plain stores
                    int dst_row = valid ? args.row_slot[t.m0 + row] : 0;
                    float *obase = args.out_f32;
                    const bool tma = full && !args.push_dst;
                    if (args.push_dst) {
                        obase = args.push_dst[dst_row >> 24];
                        dst_row &= (1 << 24) - 1;
                    }
                    float *dst = obase + (size_t)dst_row * args.ldo + t.nt * C::BN;
#pragma unroll 1
                    for (int c = 0; c < C::BN; c += 32) {
                        float v[32];
                        uint32_t p[32];
                        tmem_ld32(taddr + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) p[i] = __float_as_uint(v[i]);
                        if (tma) store_block_scatter(stg, p, lane, &tmO, t.nt * C::BN + c, dst_row);
                        else if (valid) store_row_direct(dst + c, p);
                    }
                } else if constexpr (C::EPI == EPI_WGRAD) {
                    const bool routed = t.g < args.num_routed;
                    const int gl = routed ? t.g : t.g - args.num_routed;
                    const int grow0 = gl * args.m_tiles * BM + t.m0 + eq * 32;   // row in the [groups * M, N] view
                    constexpr int COLS = C::BN * 4 / C::EPI_WARPS;               // columns of this warp
                    const int c0 = (ew >> 2) * COLS;
                    float v[64];
                    if (t.nkb > 0) {
                        tmem_ld32(taddr + c0, *reinterpret_cast<float(*)[32]>(v));
                        tmem_ld32(taddr + c0 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                        tmem_ld_wait();
                    }
#pragma unroll 1
                    for (int c = c0; c < c0 + COLS; c += 64) {
                        uint32_t p[32];
                        if (t.nkb > 0) {
                            pack_bf16<64>(v, p);
                            if (c + 64 < c0 + COLS) {          // next block's TMEM load overlaps this block's store
                                tmem_ld32(taddr + c + 64, *reinterpret_cast<float(*)[32]>(v));
                                tmem_ld32(taddr + c + 96, *reinterpret_cast<float(*)[32]>(v + 32));
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) p[i] = 0u;
                        }
                        store_block_tile(stg, p, lane, routed ? &tmO : &tmO2, t.nt * C::BN + c, grow0);
                        if (t.nkb > 0 && c + 64 < c0 + COLS) tmem_ld_wait();
                    }
                } else if constexpr (C::EPI == EPI_DSWIGLU) {
                    const int r = t.m0 + row;
                    const int I = args.inter;
                    const int n0 = t.nt * C::BN;
                    const float w = valid ? args.row_w[r] : 0.0f;
                    const __nv_bfloat16 *gsrc = valid ? args.aux + (size_t)r * 2 * I + n0 : nullptr;
                    // slot gradient of a routed row: G = <dy, o> = <dy W_down, h>, summed here over
                    // this tile's columns (v before the routing weight) against the saved h
                    const bool routed_row = valid && t.g < args.num_routed;
                    const __nv_bfloat16 *hsrc = routed_row ? args.aux_h + (size_t)r * I + n0 : nullptr;
                    float gsum = 0.0f;
#pragma unroll 1
                    for (int c = 0; c < C::BN; c += 64) {
                        uint32_t gp[32], up[32], dgp[32], dup[32], hp[32];
                        load_row_direct(gp, gsrc ? gsrc + c : nullptr);
                        load_row_direct(up, gsrc ? gsrc + I + c : nullptr);
                        load_row_direct(hp, hsrc ? hsrc + c : nullptr);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float v[32], dg[32], du[32];
                            tmem_ld32(taddr + c + 32 * half, v);
                            tmem_ld_wait();
                            if constexpr (C::EARLY_RELEASE) {
                                if (c == C::BN - 64 && half == 1) {
                                    tc_fence_before();
                                    mbar_arrive(&acce[acc]);     // every column of the accumulator is in registers
                                }
                            }
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const uint32_t gw = gp[16 * half + (i >> 1)], uw = up[16 * half + (i >> 1)];
                                const uint32_t hw = hp[16 * half + (i >> 1)];
                                const float gi = (i & 1) ? bf16_hi(gw) : bf16_lo(gw);
                                const float ui = (i & 1) ? bf16_hi(uw) : bf16_lo(uw);
                                gsum = fmaf(v[i], (i & 1) ? bf16_hi(hw) : bf16_lo(hw), gsum);
                                const float dh = w * v[i];
                                const float sg = sigmoid_f(gi);
                                dg[i] = dh * ui * sg * (1.0f + gi * (1.0f - sg));
                                du[i] = dh * gi * sg;
                            }
                            pack_bf16<32>(dg, dgp + 16 * half);
                            pack_bf16<32>(du, dup + 16 * half);
                            if constexpr (C::MX) {
                                // MXFP8 backward: dGU quantised per 1x32 block (from fp32) for the gate/up dgrad
                                if (valid) {
                                    const int cg = n0 + c + 32 * half;
                                    mx_store_block(dg, args.out_q + (size_t)r * 2 * I + cg,
                                                   args.out_scales + (size_t)r * (2 * I / 32) + cg / 32);
                                    mx_store_block(du, args.out_q + (size_t)r * 2 * I + I + cg,
                                                   args.out_scales + (size_t)r * (2 * I / 32) + (I + cg) / 32);
                                }
                            }
                        }
                        if (full) {
                            store_block_tile(stg, dgp, lane, &tmO, n0 + c, row0);
                            store_block_tile(stg, dup, lane, &tmO, I + n0 + c, row0);
                        } else if (valid) {
                            store_row_direct(args.out + (size_t)r * 2 * I + n0 + c, dgp);
                            store_row_direct(args.out + (size_t)r * 2 * I + I + n0 + c, dup);
                        }
                    }
                    if (routed_row) args.gpart[(size_t)r * args.n_tiles + t.nt] = gsum;
                } else {   // EPI_ROUTER: fp32 partial logits of this K split
                    const int r = t.m0 + row;
#pragma unroll 1
                    for (int c = 0; c < 256; c += 32) {
                        float v[32];
                        uint32_t p[32];
                        tmem_ld32(taddr + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) p[i] = __float_as_uint(v[i]);
                        if (full) store_block_tile(stg, p, lane, &tmO, c, t.nt * args.rows_total + row0);
                        else if (valid) store_row_direct(args.out_f32 + ((size_t)t.nt * args.rows_total + r) * 256 + c, p);
                    }
                }
            }
            if constexpr (!C::EARLY_RELEASE) {
                tc_fence_before();
                mbar_arrive(&acce[acc]);
            }
            if constexpr (!C::RAGGED_K) {
                // one counter per 128-row M tile (s_gorder holds each group's first one);
                // a pair tile signals both of its M tiles once both halves are stored
                if (args.ready_role == kReadySignal) {
                    const int mt = s_gorder[tt.g] + (tt.m0 - s_off[tt.g]) / BM;
                    signal_ready(args.ready + mt, lane);
                    if (C::PAIR && tt.rows > BM) signal_ready(args.ready + mt + 1, lane);
                }
            }
            if (++acc == C::ACC_BUFS) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) {
            bulk_wait0();                        // every bulk store of this warp has completed
            fence_proxy_async_global();          // ... and is ordered before later plain accesses
        }
    }

    tc_fence_before();
    __syncthreads();
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB_s, const __grid_constant__ CUtensorMap tmO,
                        const __grid_constant__ CUtensorMap tmO2, const __grid_constant__ CUtensorMap tmO3,
                        const GemmArgs args)
{
    griddep_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::RING_BYTES);
    int *aux = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(bars) + kGemmBarBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(aux) + kGemmAuxBytes);
    if ((threadIdx.x >> 5) == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    gemm_phase<C>(smem, bars, aux, tmem_base, tmA, tmB, tmB_s, tmO, tmO2, tmO3, args);
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace mok
