// fused_bwd.cuh -- the whole backward pass as ONE persistent launch (BF16, or
// with the two data-gradient GEMMs on MXFP8 operands).
//
// The counterpart of the persistent forward (fused.cuh) for the backward of
// the layer ("Cursor åpner megakernelen som ga 41 prosent flere tokens i
// sekundet": one deterministic kernel for the MoE layer's training step, BF16
// backward among the measured passes).  One cooperative launch, one CTA per SM,
// 256 threads; phases, with the grid barriers of fused.cuh:
//
//   Q0  zero the launch's tile and readiness counters; the groups' first M tiles;
//       MXFP8: quantise dy
//   --- grid barrier
//   Q1  down dgrad GEMM with the SwiGLU-backward epilogue (dGU, slot-gradient
//       partials); each epilogue warp counts its finished tile on the M tile's
//       readiness counter
//   Q2  gate/up dgrad GEMM (dX slot rows): its producer starts an M tile once
//       every down-dgrad tile of those rows is in memory -- no barrier
//   Q3  down weight gradient: streaming kernel for groups of more than 256 rows,
//       then the resident kernel for the rest (it depends on nothing of the pass)
//       gate/up weight gradient (streaming, then resident): each CTA checks,
//       once per group, that every dGU tile of the group is in memory -- no
//       barrier
//   --- grid barrier
//   Q4  slot gradients and routing-logit gradients (one thread per token)
//   --- grid barrier
//   Q5  router-gradient partial sums and the dx sum, streamed through shared
//       memory (combine.cuh: drouter_stream, dx_stream)
//   --- grid barrier
//   Q6  router-gradient reduction
//
// Every phase runs the device code of the split schedule's kernels, so the two
// schedules give byte-identical gradients.  The resident weight-gradient phases
// use almost all of shared memory: the GEMM phases' barrier blocks and group
// tables sit inside the same region, which is safe because every phase ends
// only after the last asynchronous arrival on its barriers (the producer waits
// for the MMA's release of its last stages; see gemm_phase).
#pragma once
#include <type_traits>
#include "fused.cuh"
#include "wgrad.cuh"

namespace mok {

struct FusedBwdArgs {
    GridSync gs;
    int *status;
    int *zero;                     // tile and readiness counters zeroed in Q0
    int n_zero;
    GemmArgs g1, g2, g2r, g3, g4, g4r;   // down dgrad, down wgrad (streaming, resident), gate/up dgrad, gate/up wgrad
    int g2_units, g4_units;        // resident work units (0: no resident phase)
    // slot and router gradients
    const float *gpart;
    int n_parts;
    const int *inv_perm, *topk_idx, *offsets, *chunk_start, *perm;
    const float *topk_w, *topk_p, *router_w;
    float *dl, *partial, *drouter_w;
    const __nv_bfloat16 *x;
    int T, H, E, k, S, score_fn, chunk_rows, max_chunks;
    float routed_scale;
    // dx
    const float *dxs;
    __nv_bfloat16 *dx;
    unsigned long long *trace;     // null, or [kFusedBwdTracePoints][gridDim.x] globaltimer stamps
    const int *offsets_all;        // [G + 1] row ranges of all groups (routed, then shared)
    int *mt_base;                  // [G + 1] first M tile of each group (written in Q0)
    // MXFP8 backward: dy quantised in Q0 (1x32 blocks along H) for the down dgrad
    const __nv_bfloat16 *dy;
    uint8_t *dyq, *dys;
};

// trace points: start, end of Q0, end of the dgrads, of the down weight gradient,
// of the gate/up weight gradient, of the slot gradients, of the router partials,
// of dx, of the router-gradient reduction
constexpr int kFusedBwdTracePoints = 9;

struct FusedBwdMaps {
    CUtensorMap d1B, d1Bs, d1O;              // down dgrad: W_down (MN-major), shared, dGU out
    CUtensorMap w2B, w2O, w2O2;              // down wgrad: w*h, dW_down, dWs_down
    CUtensorMap d3A, d3B, d3Bs, d3O;         // gate/up dgrad: dGU, W_gate_up (MN-major), shared, dX slots
    CUtensorMap w4A, w4O, w4O2;              // gate/up wgrad: dGU, dW_gate_up, dWs_gate_up
};

// MXFP8 backward's data-gradient GEMMs: the down dgrad pulls dy's e4m3 rows by
// token (as the MXFP8 gate/up forward pulls x) against W_down^T quantised along
// H, with the SwiGLU-backward epilogue that also quantises dGU; the gate/up dgrad
// reads those dGU codes (as the MXFP8 down forward reads h's) against
// W_gate_up^T quantised along 2I and pushes fp32 rows
using DgradDownMX = GemmCfg<256, false, false, true, false, false, EPI_DSWIGLU, true>;
using DgradGUMX = GemmCfg<256, false, false, false, false, false, EPI_PUSH, true>;

template <bool N256, bool MX = false>
struct FusedBwdCfg {
    static_assert(!MX || N256, "the MXFP8 backward takes N = 256 tiles");
    static constexpr int BN = N256 ? 256 : 128;
    // BF16 data gradients on 256-row pair tiles (at N = 256)
    using DgradDown =
        std::conditional_t<MX, DgradDownMX, GemmCfg<BN, false, true, true, false, false, EPI_DSWIGLU, false, N256>>;
    using WgradDown = GemmCfg<BN, true, true, true, false, true, EPI_WGRAD>;
    // (the push epilogue's fp32 rows are heavy: its GEMM keeps double-buffered 128-row tiles)
    using DgradGU = std::conditional_t<MX, DgradGUMX, GemmCfg<256, false, true, false, false, false, EPI_PUSH>>;
    using WgradGU = GemmCfg<256, true, true, false, true, true, EPI_WGRAD>;
    using ResDown = WgradResCfg<true>;
    using ResGU = WgradResCfg<false>;
    static constexpr int cmax(int a, int b) { return a > b ? a : b; }
    static constexpr int GEMM_RING =
        cmax(cmax(DgradDown::RING_BYTES, WgradDown::RING_BYTES), cmax(DgradGU::RING_BYTES, WgradGU::RING_BYTES));
    // GEMM ring, then the four GEMM phases' barrier blocks and the group tables
    static constexpr int GEMM_BYTES = GEMM_RING + 4 * kGemmBarBytes + kGemmAuxBytes;
    static constexpr int REGION = cmax(GEMM_BYTES, cmax(ResDown::DATA_BYTES, ResGU::DATA_BYTES));
    // region | two resident barrier blocks | TMEM slot, barrier flag, epoch
    static constexpr int SMEM_BYTES = 1024 + REGION + 2 * ResDown::BAR_BYTES + 16;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(ResDown::BAR_BYTES == ResGU::BAR_BYTES, "barrier blocks");
    static_assert(drouter_stream_bytes(kFusedThreads, 256) <= REGION, "router-gradient stream");
    static_assert(DgradDown::THREADS <= kFusedThreads && WgradDown::THREADS <= kFusedThreads &&
                  DgradGU::THREADS <= kFusedThreads && WgradGU::THREADS <= kFusedThreads &&
                  ResDown::THREADS <= kFusedThreads && ResGU::THREADS <= kFusedThreads, "phase roles fit the launch");
};

__device__ __forceinline__ void fused_bwd_stamp(const FusedBwdArgs &a, int point)
{
    if (a.trace && threadIdx.x == 0) a.trace[static_cast<size_t>(point) * gridDim.x + blockIdx.x] = globaltimer();
}

// Q1-Q3 of a persistent backward: both dgrads and both weight gradients.  No
// barrier between the four GEMMs: a CTA moves on when a GEMM's tile counter is
// exhausted, so the next GEMM starts on SMs that the previous one's tail leaves
// idle.  The gate/up dgrad waits per M tile and the gate/up weight gradient per
// group for the down dgrad's dGU rows.  trace: stamps 2 and 3 (or null).
template <class F, bool N256>
__device__ __forceinline__ void bwd_expert_gemms(uint8_t *smem, uint64_t *gbars, int *aux, uint64_t *rbars,
                                                 uint32_t tmem_base, const FusedBwdMaps &m, const GemmArgs &g1,
                                                 const GemmArgs &g2, const GemmArgs &g2r, const GemmArgs &g3,
                                                 const GemmArgs &g4, const GemmArgs &g4r, int g2_units, int g4_units,
                                                 unsigned long long *trace)
{
    constexpr int GB = kGemmBarBytes / 8;           // uint64 per GEMM barrier block
    constexpr int RB = F::ResDown::BAR_BYTES / 8;
    auto stamp = [&](int point) {
        if (trace && threadIdx.x == 0) trace[static_cast<size_t>(point) * gridDim.x + blockIdx.x] = globaltimer();
    };
    tc_fence_after();
    gemm_phase<typename F::DgradDown>(smem, gbars, aux, tmem_base, m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1);
    tc_fence_after();
    gemm_phase<typename F::DgradGU>(smem, gbars + GB, aux, tmem_base, m.d3A, m.d3B, m.d3Bs, m.d3O, m.d3O, m.d3O, g3);
    stamp(2);
    tc_fence_after();
    gemm_phase<typename F::WgradDown>(smem, gbars + 2 * GB, aux, tmem_base, m.w2B, m.w2B, m.w2B, m.w2O, m.w2O2, m.w2O,
                                      g2);
    if constexpr (N256) {
        if (g2_units > 0) {
            tc_fence_after();
            wgrad_resident_phase<typename F::ResDown>(smem, rbars, tmem_base, m.w2B, m.w2B, m.w2O, m.w2O2, g2r);
        }
    }
    stamp(3);
    tc_fence_after();
    gemm_phase<typename F::WgradGU>(smem, gbars + 3 * GB, aux, tmem_base, m.w4A, m.w4A, m.w4A, m.w4O, m.w4O2, m.w4O,
                                    g4);
    if (g4_units > 0) {
        tc_fence_after();
        wgrad_resident_phase<typename F::ResGU>(smem, rbars + RB, tmem_base, m.w4A, m.w4A, m.w4O, m.w4O2, g4r);
    }
}

template <bool N256, bool MX>
__global__ void __launch_bounds__(kFusedThreads, 1)
    moe_bwd_fused_kernel(const __grid_constant__ FusedBwdMaps m, const __grid_constant__ FusedBwdArgs a)
{
    using F = FusedBwdCfg<N256, MX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *gbars = reinterpret_cast<uint64_t *>(smem + F::GEMM_RING);          // 4 GEMM barrier blocks
    int *aux = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(gbars) + 4 * kGemmBarBytes);
    uint64_t *rbars = reinterpret_cast<uint64_t *>(smem + F::REGION);             // 2 resident barrier blocks
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(rbars) + 2 * F::ResDown::BAR_BYTES);
    volatile int *s_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5;
    const long long gtid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long gstride = static_cast<long long>(gridDim.x) * blockDim.x;

    if (threadIdx.x == 0) reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0] = *a.gs.epoch & kEpochMask;
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned long long epoch = reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0];
    const uint32_t tmem_base = *tmem_slot;
    fused_bwd_stamp(a, 0);

    // ---------------------------------------------------------------- Q0
    for (long long i = gtid; i < a.n_zero; i += gstride) a.zero[i] = 0;
    if constexpr (MX) {
        const long long nb = static_cast<long long>(a.T) * (a.H / 32);
        for (long long b = gtid; b < nb; b += gstride) quantize_block(b, a.dy, a.dyq, a.dys, a.H / 32, 0);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // first 128-row M tile of every group (the readiness counters' index)
        int acc = 0;
        for (int g = 0; g <= a.g1.num_groups; ++g) {
            a.mt_base[g] = acc;
            if (g < a.g1.num_groups) acc += (a.offsets_all[g + 1] - a.offsets_all[g] + BM - 1) / BM;
        }
    }
    fused_bwd_stamp(a, 1);
    int nb = 0;
    bool alive = grid_sync(a.gs, epoch, nb++, true, a.status, s_flag);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.gs.epoch = (epoch + 1) & kEpochMask;

    // ---------------------------------------------------------------- Q1, Q2, Q3 (both dgrads, both weight gradients)
    if (alive) {
        bwd_expert_gemms<F, N256>(smem, gbars, aux, rbars, tmem_base, m, a.g1, a.g2, a.g2r, a.g3, a.g4, a.g4r,
                                  a.g2_units, a.g4_units, a.trace);
    } else {
        fused_bwd_stamp(a, 2);
        fused_bwd_stamp(a, 3);
    }
    fused_bwd_stamp(a, 4);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- Q4
    if (alive)
        for (long long t = gtid; t < a.T; t += gstride)
            slot_grad_token(static_cast<int>(t), a.gpart, a.n_parts, a.inv_perm, a.topk_w, a.topk_p, a.dl, a.k,
                            a.score_fn, a.routed_scale);
    fused_bwd_stamp(a, 5);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- Q5
    // router-gradient partials, then the dx sum, both streamed through the
    // region's shared memory (drouter_stream, dx_stream)
    if (alive) drouter_stream(a.x, a.dl, a.offsets, a.chunk_start, a.perm, a.partial, a.H, a.E, a.k, a.chunk_rows, smem);
    fused_bwd_stamp(a, 6);
    __syncthreads();                           // the region is free again
    if (alive) dx_stream(a.dxs, a.dl, a.topk_idx, a.router_w, a.dx, a.T, a.H, a.k, a.S, smem, F::REGION);
    fused_bwd_stamp(a, 7);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- Q6
    if (alive) drouter_reduce_stream(a.partial, a.chunk_start, a.drouter_w, a.H, a.E);
    fused_bwd_stamp(a, 8);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace mok
