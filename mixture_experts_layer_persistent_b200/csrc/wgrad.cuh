// Weight gradients of lightly loaded groups with one operand resident in shared memory.
//
// For a group g with K = rows(g) routed rows, the weight gradient is the
// per-expert contraction over those rows (the BF16 backward of the layer,
// "Cursor åpner megakernelen som ga 41 prosent flere tokens i sekundet",
// paragraph on what MoK is: one gradient per expert weight, summed over the
// tokens routed to it):
//
//   gate/up:  dW_gu[g] (2I x H) = dGU_g^T (2I x K) . x_g (K x H)      x_g gathered by token
//   down:     dW_dn[g] (H x I)  = dy_g^T  (H x K)  . (w h)_g (K x I)  dy_g gathered by token
//
// With K of a few hundred rows every 128 x 256 output tile has only a few K
// blocks, so a kernel that streams both operands per tile reads three times
// the output's bytes from L2 and stalls on tile turnover.  Here a work unit is
// (group, 256-column N slab, run of M tiles): the unit's B slab (K x 256, at
// most kResidentRows rows) is loaded into shared memory once and every M tile
// of the run streams only its A block (K x 128) through a ring.  Groups with
// more rows than that go to the streaming kernel (grouped_gemm_kernel with
// args.k_split), which processes the prefix of the rows-descending group
// order; this kernel processes the rest of that order.
//
// Both operands are MN-major in shared memory (128-byte swizzle, 64-element
// chunks 8 KB apart); exactly one of them is gathered by the pull warps, the
// other comes by TMA.  Rows past the group's end are zero in the gathered
// operand (written as zeros, not loaded) and zeroed by the MMA warp in the
// contiguous one, so each tile's sum runs over exactly the group's rows in
// ascending row order: the result is deterministic and does not depend on the
// grid.
#pragma once

#include "gemm.cuh"

namespace mok {

constexpr int kResidentRows = 192;

template <bool A_GATHER_>
struct WgradResCfg {
    static constexpr bool A_GATHER = A_GATHER_;     // down: A = dy rows gathered; gate/up: B = x rows gathered
    static constexpr bool B_GATHER = !A_GATHER_;
    static constexpr int BN = 256;
    static constexpr int KB_MAX = kResidentRows / BK;        // resident K blocks
    static constexpr int A_BYTES = BM * BK * 2;              // 128 M x 64 K, two 8 KB chunks
    static constexpr int B_KB_BYTES = BN * BK * 2;           // 256 N x 64 K, four 8 KB chunks
    static constexpr int B_BYTES = KB_MAX * B_KB_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int EPI_WARPS = 4;                      // 4 or 8 (two per TMEM lane quarter)
    static constexpr int EPI_BUFS = 4;
    static constexpr int PULL_WARPS = kPullWarps;
    static constexpr int PULL_WARP0 = 2 + EPI_WARPS;
    static constexpr int THREADS = 64 + 32 * (EPI_WARPS + PULL_WARPS);
    static constexpr int TMEM_COLS = 2 * BN;                 // two accumulators
    static constexpr int EPI_STAGE_BYTES = EPI_WARPS * EPI_BUFS * 4096;
    static constexpr int BAR_BYTES = 256;
    // the group tables (offsets, order) are read through L1, not staged: the
    // shared memory goes to the resident slab, the ring and the store staging
    static constexpr int DATA_BYTES = B_BYTES + STAGES * A_BYTES + EPI_STAGE_BYTES;
    static constexpr int SMEM_BYTES = 1024 + DATA_BYTES + BAR_BYTES + 16;
    static constexpr uint32_t IDESC = idesc_bf16(BM, BN, true, true);
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(EPI_BUFS >= 1 && EPI_BUFS <= 4, "staging buffers per warp");
    static_assert((2 * STAGES + KB_MAX + 7) * 8 <= BAR_BYTES, "barrier block");
};

struct WUnit {
    int g;          // group
    int nt;         // N slab (256 columns)
    int mt0, mt1;   // M tiles [mt0, mt1)
    int krow0;      // first sorted row of the group
    int krows;      // rows of the group
    int nkb;        // K blocks
};

__device__ __forceinline__ WUnit decode_unit(int u, const GemmArgs &a, int nbig, int m_chunks)
{
    WUnit w;
    const int per_group = a.n_tiles * m_chunks;
    const int gi = nbig + u / per_group;
    const int rem = u - (gi - nbig) * per_group;
    w.nt = rem / m_chunks;
    const int mc = rem - w.nt * m_chunks;
    w.g = __ldg(a.gorder + gi);
    w.mt0 = mc * a.m_per_unit;
    w.mt1 = min(w.mt0 + a.m_per_unit, a.m_tiles);
    w.krow0 = __ldg(a.offsets + w.g);
    w.krows = __ldg(a.offsets + w.g + 1) - w.krow0;
    w.nkb = (w.krows + BK - 1) / BK;
    return w;
}

// zero rows [valid, 64) of a 64-row MN-major block of `chunks` 8 KB chunks (one warp)
__device__ __forceinline__ void zero_tail_rows(uint8_t *blk, int chunks, int valid, int lane)
{
    const int n16 = (BK - valid) * 8;
    for (int c = 0; c < chunks; ++c) {
        uint4 *p = reinterpret_cast<uint4 *>(blk + c * 8192 + valid * 128);
        for (int i = lane; i < n16; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// One resident weight-gradient phase run by every thread of the CTA.
//   smem       1024-byte aligned: C::DATA_BYTES of resident slab, A ring and staging
//   bar_block  C::BAR_BYTES of barriers for this phase
//   tmem_base  TMEM columns [0, C::TMEM_COLS) allocated by the caller
// Starts and ends with a CTA-wide barrier.
template <class C>
__device__ __forceinline__ void wgrad_resident_phase(uint8_t *smem, uint64_t *bar_block, uint32_t tmem_base,
                                                     const CUtensorMap &tmA, const CUtensorMap &tmB,
                                                     const CUtensorMap &tmO, const CUtensorMap &tmO2,
                                                     const GemmArgs &args)
{
    uint8_t *sB = smem;                                        // resident B: KB_MAX blocks
    uint8_t *sA = sB + C::B_BYTES;                             // A ring: STAGES blocks
    uint32_t *epi_stage = reinterpret_cast<uint32_t *>(sA + C::STAGES * C::A_BYTES);
    uint64_t *afull = bar_block;
    uint64_t *aempty = afull + C::STAGES;
    uint64_t *bfull = aempty + C::STAGES;
    uint64_t *bempty = bfull + C::KB_MAX;
    uint64_t *accf = bempty + 1;
    uint64_t *acce = accf + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acce + 2);
    uint64_t *drain_bar = acce + 3;                            // MMA drain on abort

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.num_groups;
    int *status = args.status;

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < C::STAGES; ++s) {
                mbar_init(&afull[s], C::A_GATHER ? 32 * C::PULL_WARPS : 1);
                mbar_init(&aempty[s], 1);
            }
            for (int kb = 0; kb < C::KB_MAX; ++kb) mbar_init(&bfull[kb], C::B_GATHER ? 32 * C::PULL_WARPS : 1);
            mbar_init(bempty, 1);
            for (int b = 0; b < 2; ++b) {
                mbar_init(&accf[b], 1);
                mbar_init(&acce[b], 32 * C::EPI_WARPS);
            }
            mbar_init(drain_bar, 1);
            *abort_flag = 0;
            fence_barrier_init();
            if constexpr (!C::A_GATHER) tma_prefetch_desc(&tmA);
            if constexpr (!C::B_GATHER) tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmO);
            tma_prefetch_desc(&tmO2);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    fence_proxy_async_global();          // operands an earlier phase of the launch wrote
    const int nbig = count_big_groups(args.offsets, args.gorder, G, args.k_split);
    const int m_chunks = (args.m_tiles + args.m_per_unit - 1) / args.m_per_unit;
    const int total = (G - nbig) * args.n_tiles * m_chunks;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (contiguous operand)
        int stage = 0;
        uint32_t phase = 0, bphase = 0;
        int ready_g = -1;                  // last group found complete
        int fills = 0;                   // ring stages whose loads this producer issued
        uint32_t bfill = 0;              // bit kb: parity of the next fill of resident block kb
        uint32_t bfilled = 0;            // bit kb: resident block kb filled by TMA at least once
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const WUnit w = decode_unit(u, args, nbig, m_chunks);
            if (w.nkb == 0) continue;
            bool ok = true;
            if constexpr (!C::B_GATHER) {
                // resident B = rows krow0.. of the contiguous [R, N] matrix, columns of slab nt
                if (lane == 0) ok = mbar_wait(bempty, bphase ^ 1u, abort_flag, status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                bphase ^= 1u;
                for (int kb = 0; kb < w.nkb; ++kb) {
                    if (lane == 0) mbar_arrive_expect_tx(&bfull[kb], C::B_KB_BYTES);
                    __syncwarp();
                    if (lane < C::BN / 64)
                        tma_load_2d(sB + kb * C::B_KB_BYTES + lane * 8192, &tmB, &bfull[kb], w.nt * C::BN + lane * 64,
                                    w.krow0 + kb * BK);
                    bfill ^= 1u << kb;
                    bfilled |= 1u << kb;
                }
            } else {
                if (args.ready_role == kReadyWaitGroup && w.g != ready_g) {
                    // the group's A rows come from an earlier phase of the launch
                    ok = wait_group_ready(args, w.g, lane, abort_flag, status);
                    ready_g = w.g;
                    if (!ok) break;
                }
                // A = rows krow0.. of the contiguous [R, M] matrix, columns of M tile mt
                for (int mt = w.mt0; mt < w.mt1 && ok; ++mt) {
                    for (int kb = 0; kb < w.nkb; ++kb) {
                        if (lane == 0) {
                            ok = mbar_wait(&aempty[stage], phase ^ 1u, abort_flag, status);
                            if (ok) mbar_arrive_expect_tx(&afull[stage], C::A_BYTES);
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        if (lane < BM / 64)
                            tma_load_2d(sA + stage * C::A_BYTES + lane * 8192, &tmA, &afull[stage], mt * BM + lane * 64,
                                        w.krow0 + kb * BK);
                        ++fills;
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (!ok) break;
            }
        }
        if (lane == 0) {
            // the last fills: after an abort, let their loads land (bounded) before the CTA
            // releases its shared memory; otherwise wait until the MMA has released them, so
            // that no arrival on this phase's barriers is still in flight when it ends
            const bool aborted = *abort_flag != 0;
            int s2 = stage;
            uint32_t ph = phase;
            for (int i = 0; i < min(fills, C::STAGES); ++i) {
                if (--s2 < 0) {
                    s2 = C::STAGES - 1;
                    ph ^= 1u;
                }
                mbar_drain(aborted ? &afull[s2] : &aempty[s2], ph);
            }
            if (aborted) {
                for (int kb = 0; kb < C::KB_MAX; ++kb)
                    if (bfilled & (1u << kb)) mbar_drain(&bfull[kb], ((bfill >> kb) & 1u) ^ 1u);
            } else if (bfilled) {
                mbar_drain(bempty, bphase ^ 1u);      // the resident block of the last unit released
            }
        }
    } else if (warp >= C::PULL_WARP0) {
        // ------------------------------------------------------------ pull warps (gathered operand)
        // Thread p copies 16-byte column c16 of rows r0 + RS i (i < NR) of every
        // 64-row K block; a row's token index is the same for every M tile of
        // the unit, so the indices are read once per unit.
        constexpr int RS = 32 * C::PULL_WARPS / 8;     // a thread's rows are RS apart
        constexpr int NR = BK / RS;                    // rows per thread and K block
        const int p = threadIdx.x - 32 * C::PULL_WARP0;
        const int c16 = p & 7;
        const int r0 = p >> 3;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(args.gather_src);
        const size_t ld = static_cast<size_t>(args.gather_ld) * 2;
        int stage = 0;
        uint32_t phase = 0, bphase = 0;
        int pfills = 0;                  // A ring stages these warps filled
        bool pfilled = false;            // resident block filled at least once
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const WUnit w = decode_unit(u, args, nbig, m_chunks);
            if (w.nkb == 0) continue;
            int tok[C::KB_MAX][NR];
#pragma unroll
            for (int kb = 0; kb < C::KB_MAX; ++kb)
#pragma unroll
                for (int i = 0; i < NR; ++i) {
                    const int kr = kb * BK + r0 + RS * i;
                    tok[kb][i] = kr < w.krows ? __ldg(args.row_token + w.krow0 + kr) : -1;
                }
            if constexpr (C::B_GATHER) {
                ok = mbar_wait(bempty, bphase ^ 1u, abort_flag, status);
                if (!ok) break;
                bphase ^= 1u;
                pfilled = true;
#pragma unroll
                for (int kb = 0; kb < C::KB_MAX; ++kb) {
                    if (kb >= w.nkb) break;
                    uint8_t *dst = sB + kb * C::B_KB_BYTES;
#pragma unroll
                    for (int i = 0; i < NR; ++i) {
                        const int r = r0 + RS * i;
                        uint8_t *d = dst + r * 128 + ((c16 ^ (r & 7)) << 4);
                        if (tok[kb][i] >= 0) {
                            const uint8_t *row = src + tok[kb][i] * ld + (w.nt * C::BN) * 2 + c16 * 16;
#pragma unroll
                            for (int j = 0; j < C::BN / 64; ++j) cp_async16(d + j * 8192, row + j * 128);
                        } else {
#pragma unroll
                            for (int j = 0; j < C::BN / 64; ++j)
                                *reinterpret_cast<uint4 *>(d + j * 8192) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    fence_proxy_async_smem();
                    cp_async_arrive_noinc(&bfull[kb]);
                }
            } else {
                for (int mt = w.mt0; mt < w.mt1 && ok; ++mt) {
#pragma unroll
                    for (int kb = 0; kb < C::KB_MAX; ++kb) {
                        if (kb >= w.nkb) break;
                        ok = mbar_wait(&aempty[stage], phase ^ 1u, abort_flag, status);
                        if (!ok) break;
                        uint8_t *dst = sA + stage * C::A_BYTES;
#pragma unroll
                        for (int i = 0; i < NR; ++i) {
                            const int r = r0 + RS * i;
                            uint8_t *d = dst + r * 128 + ((c16 ^ (r & 7)) << 4);
                            if (tok[kb][i] >= 0) {
                                const uint8_t *row = src + tok[kb][i] * ld + (mt * BM) * 2 + c16 * 16;
#pragma unroll
                                for (int j = 0; j < BM / 64; ++j) cp_async16(d + j * 8192, row + j * 128);
                            } else {
#pragma unroll
                                for (int j = 0; j < BM / 64; ++j)
                                    *reinterpret_cast<uint4 *>(d + j * 8192) = make_uint4(0u, 0u, 0u, 0u);
                            }
                        }
                        fence_proxy_async_smem();
                        cp_async_arrive_noinc(&afull[stage]);
                        ++pfills;
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        }
        cp_async_wait_all();             // nothing of this thread still lands in shared memory
        if (p == 0 && !*abort_flag) {
            // what the pull warps filled last has been released by the MMA (see the producer)
            if constexpr (C::B_GATHER) {
                if (pfilled) mbar_drain(bempty, bphase ^ 1u);
            } else {
                int s2 = stage;
                uint32_t ph = phase;
                for (int i = 0; i < min(pfills, C::STAGES); ++i) {
                    if (--s2 < 0) {
                        s2 = C::STAGES - 1;
                        ph ^= 1u;
                    }
                    mbar_drain(&aempty[s2], ph);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0, bph = 0;     // bph: parity bit of bfull[kb]
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const WUnit w = decode_unit(u, args, nbig, m_chunks);
            for (int mt = w.mt0; mt < w.mt1; ++mt) {
                if (lane == 0) ok = mbar_wait(&acce[acc], acc_phase ^ 1u, abort_flag, status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
                for (int kb = 0; kb < w.nkb; ++kb) {
                    const int valid = w.krows - kb * BK;
                    if (mt == w.mt0) {
                        // first use of resident block kb in this unit
                        if (lane == 0) ok = mbar_wait(&bfull[kb], (bph >> kb) & 1u, abort_flag, status);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        bph ^= 1u << kb;
                        if constexpr (!C::B_GATHER) {
                            if (valid < BK) {
                                zero_tail_rows(sB + kb * C::B_KB_BYTES, C::BN / 64, valid, lane);
                                fence_proxy_async_smem();
                                __syncwarp();
                            }
                        }
                    }
                    if (lane == 0) ok = mbar_wait(&afull[stage], phase, abort_flag, status);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t *a_blk = sA + stage * C::A_BYTES;
                    if constexpr (!C::A_GATHER) {
                        if (valid < BK) {
                            zero_tail_rows(a_blk, BM / 64, valid, lane);
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        fence_proxy_async_smem();          // cp.async data -> tensor core
                        const uint32_t a0 = smem_u32(a_blk), b0 = smem_u32(sB + kb * C::B_KB_BYTES);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            umma_bf16(d_tmem, smem_desc_sw128(a0 + k * 2048, 8192, 1024),
                                      smem_desc_sw128(b0 + k * 2048, 8192, 1024), C::IDESC, (kb | k) != 0 ? 1u : 0u);
                        umma_commit(&aempty[stage]);
                    }
                    __syncwarp();
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) {
                    if (w.nkb > 0) umma_commit(&accf[acc]);
                    else mbar_arrive(&accf[acc]);
                }
                __syncwarp();
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every MMA of the unit has been issued: the resident block is free once they complete
            if (ok && w.nkb > 0 && lane == 0) umma_commit(bempty);
            __syncwarp();
        }
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
            // the MMAs this warp issued complete before TMEM is released
            if (lane == 0) {
                umma_commit(drain_bar);
                mbar_drain(drain_bar, 0);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue: fp32 TMEM -> bf16 dW tiles
        const int eq = warp & 3;
        const int ew = warp - 2;
        EpiStage stg{reinterpret_cast<uint32_t *>(epi_stage) + ew * C::EPI_BUFS * 1024, C::EPI_BUFS, 0};
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
            const WUnit w = decode_unit(u, args, nbig, m_chunks);
            const bool routed = w.g < args.num_routed;
            const int gl = routed ? w.g : w.g - args.num_routed;
            for (int mt = w.mt0; mt < w.mt1; ++mt) {
                ok = mbar_wait(&accf[acc], acc_phase, abort_flag, status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * C::BN) + (static_cast<uint32_t>(eq * 32) << 16);
                const int grow0 = gl * args.m_tiles * BM + mt * BM + eq * 32;
                constexpr int COLS = C::BN * 4 / C::EPI_WARPS;       // columns of this warp
                const int c0 = (ew >> 2) * COLS;
                float v[64];
                if (w.nkb > 0) {
                    tmem_ld32(taddr + c0, *reinterpret_cast<float(*)[32]>(v));
                    tmem_ld32(taddr + c0 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                    tmem_ld_wait();
                }
#pragma unroll 1
                for (int c = c0; c < c0 + COLS; c += 64) {
                    uint32_t pk[32];
                    if (w.nkb > 0) {
                        pack_bf16<64>(v, pk);
                        if (c + 64 < c0 + COLS) {          // next block's TMEM load overlaps this block's store
                            tmem_ld32(taddr + c + 64, *reinterpret_cast<float(*)[32]>(v));
                            tmem_ld32(taddr + c + 96, *reinterpret_cast<float(*)[32]>(v + 32));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) pk[i] = 0u;
                    }
                    store_block_tile(stg, pk, lane, routed ? &tmO : &tmO2, w.nt * C::BN + c, grow0);
                    if (w.nkb > 0 && c + 64 < c0 + COLS) tmem_ld_wait();
                }
                tc_fence_before();
                mbar_arrive(&acce[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        if (lane == 0) {
            bulk_wait0();
            fence_proxy_async_global();
        }
    }

    tc_fence_before();
    __syncthreads();
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    wgrad_resident_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                          const GemmArgs args)
{
    griddep_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::DATA_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(bars) + C::BAR_BYTES);
    if ((threadIdx.x >> 5) == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    wgrad_resident_phase<C>(smem, bars, tmem_base, tmA, tmB, tmO, tmO2, args);
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace mok
