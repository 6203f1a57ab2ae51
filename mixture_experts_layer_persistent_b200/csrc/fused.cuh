// fused.cuh -- the whole forward pass of the layer as ONE persistent launch.
//
// "Mixture-of-Kittens" fuses the MoE layer's communication and computation
// into a single deterministic kernel ("Cursor åpner megakernelen som ga 41
// prosent flere tokens i sekundet", the quoted paragraph; "Cursor
// veröffentlicht MoE-Megakernel Mixture-of-Kittens als Open Source",
// introduction), so that nothing between the layer's steps waits on the CPU
// ("Kommunikation im Kernel").  On one B200 the steps become phases of one
// cooperative launch, one CTA per SM, 256 threads (the GEMM roles: TMA
// producer, MMA issuer, four epilogue warps, two pull warps):
//
//   P0  zero the launch's counters; split the router weights into three bf16
//       terms; MXFP8: quantise x
//   --- grid barrier
//   P1  router GEMM (tensor cores, split over K)
//   --- grid barrier
//   P2  scores and top-k, one warp per token; each selection is also counted
//       in its dispatch chunk's histogram (integer atomics)
//   --- grid barrier
//   P3  per dispatch chunk: scan of the histograms and stable placement of the
//       chunk's (token, slot) rows (every CTA derives its own chunk's base rows)
//   --- grid barrier
//   P4  gate/up GEMM with the SwiGLU epilogue, then the down GEMM with the push
//       epilogue.  No barrier between them: each gate/up epilogue warp counts
//       its finished tile on the M tile's readiness counter, and the down
//       GEMM's producer starts a tile only once every gate/up tile of those
//       rows is in memory.  A CTA moves to the down GEMM as soon as the gate/up
//       tiles are all claimed and its own are done (the fine-grained
//       dependency idea of "Megakernels are dead and back…", the case against
//       megakernels: tile-level triggers instead of a kernel boundary).
//   --- grid barrier
//   P5  fixed-order combine of the slot rows, streamed through shared memory
//       (combine.cuh: combine_stream)
//
// The phases run the same device code as the separate kernels of the split
// schedule, so both schedules give byte-identical results.
//
// Grid barrier.  Arrival tags carry a marker byte and a launch epoch kept in the
// pass's buffer: every CTA reads the epoch once at the start, CTA 0 advances it
// right after the first barrier (when every CTA has read it), so a stale tag of
// an earlier launch (or of a CUDA-graph replay) never matches, leftover memory
// lacks the marker, and nothing has to be zeroed before the launch.  Each CTA publishes its tag; CTA 0 waits (bounded) for
// every tag and then publishes the release tag, which every CTA waits for
// (bounded).  A CTA whose barrier wait runs out records MOK_STATUS_TIMEOUT and
// skips the rest of the work (still arriving at the later barriers), so a
// failure never leaves the kernel running or touching memory past its inputs.
#pragma once
#include "combine.cuh"
#include "gemm.cuh"
#include "quant.cuh"
#include "route.cuh"

namespace mok {

constexpr int kFusedThreads = 64 + 32 * (4 + kPullWarps);   // the GEMM roles: 8 warps
constexpr int kMaxFusedCtas = 1024;
// Above any phase's own bounded waits (a CTA stops waiting after its first
// 2 s timeout in a phase, and P4 holds two phases).
constexpr uint64_t kGridSyncLimitNs = 10000000000ull;
// Tag of barrier b of a launch: marker byte | 48-bit epoch | b + 1.  The marker
// keeps leftover memory from reading as a tag: the words of a buffer's first use
// hold whatever was there (all-ones, from an int array of -1s, would otherwise
// read as every barrier reached), and a word matches only with the marker byte,
// the launch's epoch and a barrier index at least b + 1.
constexpr unsigned long long kEpochMask = (1ull << 48) - 1;
constexpr unsigned long long kTagMarker = 0xA5ull;

struct GridSync {
    unsigned long long *flags;     // [gridDim.x] arrival tag of each CTA
    unsigned long long *go;        // release tag written by CTA 0
    unsigned long long *epoch;     // launch epoch (read at start, advanced after barrier 0)
};

struct FusedFwdArgs {
    GridSync gs;
    int *status;
    int *zero;                     // counters zeroed in P0: tile counters, readiness, histograms
    int n_zero;
    // P0
    const float *router_w;
    __nv_bfloat16 *wr3;
    int *all_rows;
    int T, H, E, k, S;
    const __nv_bfloat16 *x;        // MXFP8: quantised into xq, xs
    uint8_t *xq, *xs;
    __nv_bfloat16 *xdq;            // MXFP8 training: the dequantised x (or null)
    // P1-P4
    GemmArgs gr, ga, gd;
    SelectArgs sa;
    DispatchArgs da;
    int n_chunks;
    // P5
    const void *O;                 // slot rows: fp32 (BF16 layer) or bf16 (MXFP8 layer)
    __nv_bfloat16 *y;
    unsigned long long *trace;     // null, or [kFusedTracePoints][gridDim.x] globaltimer stamps
};

// trace points: start, then the end of P0, P1, P2, P3, gate/up, down, P5; the
// ninth repeats the end (the backward has one point more)
constexpr int kFusedTracePoints = 9;

struct FusedMaps {
    CUtensorMap rA, rB, rO;                  // router GEMM
    CUtensorMap gB, gBs, gO, gO2, gO3;       // gate/up GEMM
    CUtensorMap dA, dB, dBs, dO;             // down GEMM
};

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long barrier_tag(unsigned long long epoch, int b)
{
    return (kTagMarker << 56) | (epoch << 8) | static_cast<unsigned long long>(b + 1);
}

// reached when the marker and the epoch match and the barrier index is b or later
__device__ __forceinline__ bool tag_reached(unsigned long long v, unsigned long long epoch, int b)
{
    return (v >> 56) == kTagMarker && ((v >> 8) & kEpochMask) == epoch && static_cast<int>(v & 0xFFu) >= b + 1;
}

// Barrier b of the launch.  Returns whether this CTA is still alive.
__device__ __forceinline__ bool grid_sync(const GridSync &gs, unsigned long long epoch, int b, bool alive,
                                          int *status, volatile int *s_flag)
{
    __syncthreads();                                 // the CTA's work of the phase is issued and done
    const unsigned long long tag = barrier_tag(epoch, b);
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        __threadfence();
        st_release_gpu_u64(&gs.flags[blockIdx.x], tag);
        *s_flag = alive ? 1 : 0;
    }
    if (alive) {
        if (blockIdx.x == 0 && threadIdx.x < 32) {
            bool ok = true;
            const uint64_t t0 = globaltimer();
            for (int i = lane; i < static_cast<int>(gridDim.x) && ok; i += 32)
                while (!tag_reached(ld_acquire_gpu_u64(&gs.flags[i]), epoch, b))
                    if (globaltimer() - t0 > kGridSyncLimitNs) {
                        ok = false;
                        break;
                    }
            ok = __all_sync(0xffffffffu, ok);
            if (lane == 0) {
                if (ok) {
                    __threadfence();
                    st_release_gpu_u64(gs.go, tag);
                } else {
                    atomicOr(status, kStatusTimeout);
                    *s_flag = 0;
                }
            }
        }
        if (threadIdx.x == 0 && *s_flag) {
            const uint64_t t0 = globaltimer();
            while (!tag_reached(ld_acquire_gpu_u64(gs.go), epoch, b))
                if (globaltimer() - t0 > kGridSyncLimitNs) {
                    atomicOr(status, kStatusTimeout);
                    *s_flag = 0;
                    break;
                }
            __threadfence();
        }
    }
    __syncthreads();
    const bool ok = *s_flag != 0;
    __syncthreads();
    return ok;
}

__device__ __forceinline__ void fused_stamp(const FusedFwdArgs &a, int point)
{
    if (a.trace && threadIdx.x == 0) a.trace[static_cast<size_t>(point) * gridDim.x + blockIdx.x] = globaltimer();
}

template <bool MX>
struct FusedCfg {
    using Router = GemmCfg<256, false, false, false, false, false, EPI_ROUTER>;
    // BF16 gate/up: 256-row pair tiles (MXFP8 keeps 128-row tiles: its block scales take
    // TMEM columns); the down GEMM's push epilogue is heavy, so it keeps double-buffered
    // 128-row tiles
    using GateUp = GemmCfg<256, false, false, true, false, false, EPI_SWIGLU, MX, !MX>;
    using Down = GemmCfg<256, false, false, false, false, false, EPI_PUSH, MX>;
    static constexpr int cmax(int a, int b) { return a > b ? a : b; }
    static constexpr int RING = cmax(Router::RING_BYTES, cmax(GateUp::RING_BYTES, Down::RING_BYTES));
    // ring | three barrier blocks (one per GEMM phase) | group tables | TMEM slot, barrier flag
    static constexpr int SMEM_BYTES = 1024 + RING + 3 * kGemmBarBytes + kGemmAuxBytes + 16;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(Router::THREADS <= kFusedThreads && GateUp::THREADS <= kFusedThreads &&
                  Down::THREADS <= kFusedThreads, "phase roles fit the launch");
    // routing phases use the ring's memory: select rows, dispatch masks and tables
    static_assert(kFusedThreads / 32 * 256 * 4 <= RING && (256 * kMaskWords + 512) * 4 <= RING, "routing scratch");
};

template <bool MX>
__global__ void __launch_bounds__(kFusedThreads, 1)
    moe_fwd_fused_kernel(const __grid_constant__ FusedMaps m, const __grid_constant__ FusedFwdArgs a)
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

    // the launch epoch, read once by every CTA before its first arrival
    if (threadIdx.x == 0) reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0] = *a.gs.epoch & kEpochMask;
    if (warp == 1) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned long long epoch = reinterpret_cast<volatile unsigned long long *>(tmem_slot + 2)[0];
    const uint32_t tmem_base = *tmem_slot;
    fused_stamp(a, 0);

    // ---------------------------------------------------------------- P0
    for (long long i = gtid; i < a.n_zero; i += gstride) a.zero[i] = 0;
    if (gtid == 0) {
        a.all_rows[0] = 0;
        a.all_rows[1] = a.T;
    }
    for (long long i = gtid; i < static_cast<long long>(a.E) * a.H; i += gstride) router_split_elem(i, a.router_w, a.wr3, a.H);
    if constexpr (MX) {
        const long long nb = static_cast<long long>(a.T) * a.H / 32;
        for (long long b = gtid; b < nb; b += gstride) quantize_block(b, a.x, a.xq, a.xs, a.H / 32, 0, a.xdq);
    }
    fused_stamp(a, 1);
    int nb = 0;                                      // barriers passed
    bool alive = grid_sync(a.gs, epoch, nb++, true, a.status, s_flag);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.gs.epoch = (epoch + 1) & kEpochMask;   // every CTA has read it

    // ---------------------------------------------------------------- P1
    if (alive)
        gemm_phase<typename F::Router>(smem, bars, aux, tmem_base, m.rA, m.rB, m.rB, m.rO, m.rO, m.rO, a.gr);
    fused_stamp(a, 2);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- P2
    if (alive) {
        float *row = reinterpret_cast<float *>(smem) + warp * 256;
        const int nw = kFusedThreads / 32;
        for (int t = blockIdx.x * nw + warp; t < a.T; t += gridDim.x * nw) select_token(a.sa, t, lane, row);
    }
    fused_stamp(a, 3);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- P3
    if (alive) {
        uint32_t(*s_mask)[kMaskWords] = reinterpret_cast<uint32_t(*)[kMaskWords]>(smem);
        int *s_base = reinterpret_cast<int *>(smem) + 256 * kMaskWords;
        int *s_cnt = s_base + 256;
        for (int c = blockIdx.x; c < a.n_chunks; c += gridDim.x)
            dispatch_scan_place_chunk(a.da, c, a.n_chunks, c == 0, s_mask, s_base, s_cnt);
    }
    fused_stamp(a, 4);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- P4
    if (alive) {
        gemm_phase<typename F::GateUp>(smem, bars + kGemmBarBytes / 8, aux, tmem_base, m.gB, m.gB, m.gBs, m.gO, m.gO2,
                                       m.gO3, a.ga);
        fused_stamp(a, 5);
        tc_fence_after();
        gemm_phase<typename F::Down>(smem, bars + 2 * kGemmBarBytes / 8, aux, tmem_base, m.dA, m.dB, m.dBs, m.dO, m.dO,
                                     m.dO, a.gd);
    } else {
        fused_stamp(a, 5);
    }
    fused_stamp(a, 6);
    alive = grid_sync(a.gs, epoch, nb++, alive, a.status, s_flag);

    // ---------------------------------------------------------------- P5
    // (the GEMM ring's shared memory streams the slot rows: combine_stream)
    if (alive) {
        if constexpr (MX)
            combine_stream<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(a.O), a.sa.topk_w, a.y, a.T, a.H, a.k,
                                          a.S, smem, F::RING);
        else
            combine_stream<float>(static_cast<const float *>(a.O), a.sa.topk_w, a.y, a.T, a.H, a.k, a.S, smem,
                                  F::RING);
    }
    fused_stamp(a, 7);
    fused_stamp(a, 8);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace mok
