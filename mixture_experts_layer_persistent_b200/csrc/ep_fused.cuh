// ep_fused.cuh -- an expert-parallel owner's experts phase as ONE persistent launch.
//
// The same steps as the split launches of the phase (ep.cuh, then the two
// grouped GEMMs), as phases of one cooperative launch with the persistent
// forward's roles and grid barrier (fused.cuh):
//
//   E0  zero the launch's tile and readiness counters; CTA 0 builds the owner's
//       group ranges and group order (ep_layout_block) and the list of token rows
//       it receives (ep_unique_block)
//   --- grid barrier
//   E1  the owner's sorted-row maps (ep_rows_block, CTAs over segments) and the
//       pull of every received token row (all warps; x rows, or x's MXFP8 codes
//       and scales)
//   --- grid barrier
//   E2  gate/up GEMM with the SwiGLU epilogue, then the down GEMM whose push
//       epilogue stores each row into the slot rows of the token's rank; no
//       barrier between them (per-M-tile readiness, as in the persistent forward)
//
// "Kommunikation im Kernel" ("Cursor veröffentlicht MoE-Megakernel
// Mixture-of-Kittens als Open Source"): the pull and the push happen inside the
// launch.  Every phase calls the device functions of the split launches, so the
// two schedules give byte-identical results.
#pragma once
#include "ep.cuh"
#include "fused.cuh"
#include "fused_bwd.cuh"

namespace mok {

struct EpFusedArgs {
    GridSync gs;
    int *status;
    int *zero;                     // counters zeroed in E0: tile counters, then readiness counters
    int n_zero;
    EpView v;
    EpArgs ea;
    EpPull pull[2];                // BF16: x rows; MXFP8: x codes, x scales
    int n_pull;
    int pull16[2];                 // 1: 16-byte units, 0: 8-byte units
    GemmArgs ga, gd;
};

template <bool MX>
__global__ void __launch_bounds__(kFusedThreads, 1)
    moe_ep_experts_fused_kernel(const __grid_constant__ FusedMaps m, const __grid_constant__ EpFusedArgs a)
{
    using F = FusedCfg<MX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + F::RING);
    int *aux = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(bars) + 3 * kGemmBarBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(aux) + kGemmAuxBytes);
    volatile int *s_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gtid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long gstride = static_cast<long long>(gridDim.x) * blockDim.x;

    if (threadIdx.x == 0) reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0] = *a.gs.epoch & kEpochMask;
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned long long epoch = reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0];
    const uint32_t tmem_base = *tmem_slot;

    // ---------------------------------------------------------------- E0
    for (long long i = gtid; i < a.n_zero; i += gstride) a.zero[i] = 0;
    if (blockIdx.x == 0) {
        int *scratch = reinterpret_cast<int *>(smem);          // the GEMM ring is free until E2
        ep_layout_block(a.v, a.ea, scratch);
        __syncthreads();
        ep_unique_block(a.v, a.ea, scratch + 1024);
    }
    int nb = 0;
    bool alive = grid_sync(a.gs, epoch, nb++, true, a.status, s_flag);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.gs.epoch = (epoch + 1) & kEpochMask;   // every CTA has read it

    // ---------------------------------------------------------------- E1
    if (alive) {
        const int n_rb = ep_row_blocks(a.ea);
        for (int b = blockIdx.x; b < n_rb; b += gridDim.x) ep_rows_block(a.v, a.ea, b);
        const int gw = static_cast<int>(gtid >> 5), nw = static_cast<int>(gstride >> 5);
        for (int q = 0; q < a.n_pull; ++q) {
            if (a.pull16[q]) ep_pull_rows<uint4>(a.pull[q], gw, nw, lane);
            else ep_pull_rows<uint2>(a.pull[q], gw, nw, lane);
        }
    }
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- E2
    if (alive) {
        gemm_phase<typename F::GateUp>(smem, bars + kGemmBarBytes / 8, aux, tmem_base, m.gB, m.gB, m.gBs, m.gO, m.gO2,
                                       m.gO3, a.ga);
        tc_fence_after();
        gemm_phase<typename F::Down>(smem, bars + 2 * kGemmBarBytes / 8, aux, tmem_base, m.dA, m.dB, m.dBs, m.dO, m.dO,
                                     m.dO, a.gd);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// The owner's backward experts phase as one persistent launch:
//
//   B0  zero the launch's counters; the per-rank dX and slot-gradient tables; the
//       first 128-row M tile of every group; the pull of the dy rows (all warps)
//   --- grid barrier
//   B0b MXFP8 only: the pulled dy rows quantised, the pulled x codes decoded
//       (ep_mx_prepare)
//   --- grid barrier (MXFP8 only)
//   B1  down dgrad, gate/up dgrad (its push epilogue stores each dX row into the
//       dX slot rows of the token's rank), both weight gradients: the persistent
//       backward's GEMM phases (bwd_expert_gemms), with their per-tile readiness
//   --- grid barrier
//   B2  the slot-gradient partials of every routed row pushed to its token's rank
struct EpBwdFusedArgs {
    GridSync gs;
    int *status;
    int *zero;
    int n_zero;
    EpPull pull;                   // dy rows
    int pull16;
    EpTable tdx, tg;               // every rank's dX slot rows and slot-gradient partials
    float **push_dx, **push_g;     // their device tables (the push epilogue and B2 read them)
    int world;
    GemmArgs g1, g2, g2r, g3, g4, g4r;
    int g2_units, g4_units;
    const int *offsets_all;        // [G + 1] the owner's group ranges
    int *mt_base;                  // [G + 1] first 128-row M tile of each group (written in B0)
    const float *gpart;            // the owner's slot-gradient partials, [routed rows, nt]
    const int *row_gdst, *seg;
    int n_seg, nt, tk;
    EpMxPrep prep;                 // MXFP8: dy quantised and x decoded after the pull (B0b)
};

template <bool N256, bool MX>
__global__ void __launch_bounds__(kFusedThreads, 1)
    moe_ep_bwd_experts_fused_kernel(const __grid_constant__ FusedBwdMaps m, const __grid_constant__ EpBwdFusedArgs a)
{
    using F = FusedBwdCfg<N256, MX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *gbars = reinterpret_cast<uint64_t *>(smem + F::GEMM_RING);
    int *aux = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(gbars) + 4 * kGemmBarBytes);
    uint64_t *rbars = reinterpret_cast<uint64_t *>(smem + F::REGION);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(rbars) + 2 * F::ResDown::BAR_BYTES);
    volatile int *s_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gtid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long gstride = static_cast<long long>(gridDim.x) * blockDim.x;

    if (threadIdx.x == 0) reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0] = *a.gs.epoch & kEpochMask;
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned long long epoch = reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0];
    const uint32_t tmem_base = *tmem_slot;

    // ---------------------------------------------------------------- B0
    for (long long i = gtid; i < a.n_zero; i += gstride) a.zero[i] = 0;
    if (gtid < a.world) {
        a.push_dx[gtid] = a.tdx.p[gtid];
        a.push_g[gtid] = a.tg.p[gtid];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        int acc = 0;
        for (int g = 0; g <= a.g1.num_groups; ++g) {
            a.mt_base[g] = acc;
            if (g < a.g1.num_groups) acc += (a.offsets_all[g + 1] - a.offsets_all[g] + BM - 1) / BM;
        }
    }
    if (a.pull16) ep_pull_rows<uint4>(a.pull, static_cast<int>(gtid >> 5), static_cast<int>(gstride >> 5), lane);
    else ep_pull_rows<uint2>(a.pull, static_cast<int>(gtid >> 5), static_cast<int>(gstride >> 5), lane);
    int nb = 0;
    bool alive = grid_sync(a.gs, epoch, nb++, true, a.status, s_flag);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.gs.epoch = (epoch + 1) & kEpochMask;   // every CTA has read it

    // ---------------------------------------------------------------- B0b (MXFP8)
    if constexpr (MX) {
        if (alive) ep_mx_prepare(a.prep, gtid, gstride);
        alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);
    }

    // ---------------------------------------------------------------- B1
    if (alive)
        bwd_expert_gemms<F, N256>(smem, gbars, aux, rbars, tmem_base, m, a.g1, a.g2, a.g2r, a.g3, a.g4, a.g4r,
                                  a.g2_units, a.g4_units, nullptr);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- B2
    if (alive) ep_push_gpart(a.gpart, a.row_gdst, a.seg, a.n_seg, a.nt, a.push_g, a.world, a.tk, a.status, gtid, gstride);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace mok
