// mok.cu -- the C ABI of libmok (see include/mok.h): argument checks, the
// layout of the caller's ctx/scratch buffers, TMA descriptors and the launch
// sequence of the forward and backward passes.  All launches go to the
// caller's stream; nothing here waits on the device except moe_status and the
// host-buffer variants.
#include "mok.h"

#include <cudaTypedefs.h>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "combine.cuh"
#include "ep.cuh"
#include "ep_fused.cuh"
#include "fused.cuh"
#include "fused_bwd.cuh"
#include "gemm.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "wgrad.cuh"

namespace mok {

__device__ int g_status;   // device status word (MOK_STATUS_* bits)

// Scratch of moe_fwd_static: the library's own storage, so that callers who
// cannot allocate still get a forward pass.  Host code must not use the symbol
// itself as a pointer; it looks up the device address once per device.
static __device__ __align__(256) unsigned char g_static_scratch[MOK_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kChunkRows = 256;   // router-gradient row chunk
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    bool ok = false;
    int sms = 0;
    int *status = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// per-thread description of the last failure (moe_last_error)
thread_local char t_last_error[256] = "";

int fail(int code, const char *what, cudaError_t e = cudaSuccess)
{
    if (e != cudaSuccess)
        snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%s)", what, cudaGetErrorString(e),
                 cudaGetErrorName(e));
    else
        snprintf(t_last_error, sizeof(t_last_error), "%s", what);
    return code;
}

// per-thread phase tracing (moe_trace_events)
thread_local cudaEvent_t t_fwd_ev[MOK_FWD_PHASES + 1];
thread_local cudaEvent_t t_bwd_ev[MOK_BWD_PHASES + 1];
thread_local bool t_fwd_on = false, t_bwd_on = false;
thread_local int t_drop_signal = 0;     // moe_test_drop_signal
thread_local int t_schedule = MOK_SCHEDULE_PERSISTENT;   // moe_set_schedule
thread_local unsigned long long *t_dev_trace = nullptr;   // moe_trace_device (forward)
thread_local size_t t_dev_trace_bytes = 0;
thread_local unsigned long long *t_dev_trace_bwd = nullptr;   // moe_trace_device (backward)
thread_local size_t t_dev_trace_bwd_bytes = 0;
thread_local int t_launches = 0;        // kernels launched by the current / last forward or backward
thread_local bool t_pdl = false;        // launches of the current pass use programmatic dependent launch

inline int mark_fwd(int i, cudaStream_t s)
{
    if (!t_fwd_on) return MOK_OK;
    const cudaError_t e = cudaEventRecord(t_fwd_ev[i], s);
    return e == cudaSuccess ? MOK_OK : fail(MOK_ERR_LAUNCH, "cudaEventRecord(trace event)", e);
}
inline int mark_bwd(int i, cudaStream_t s)
{
    if (!t_bwd_on) return MOK_OK;
    const cudaError_t e = cudaEventRecord(t_bwd_ev[i], s);
    return e == cudaSuccess ? MOK_OK : fail(MOK_ERR_LAUNCH, "cudaEventRecord(trace event)", e);
}

const DeviceInfo *device_info()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.init) {
        d.init = true;
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        void *p = nullptr;
        const bool sym = cudaGetSymbolAddress(&p, g_status) == cudaSuccess;
        d.status = static_cast<int *>(p);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        d.ok = major == 10 && minor == 0 && sym && g_encode != nullptr && d.sms > 0;
    }
    return d.ok ? &d : nullptr;
}

// 2D tensor map over a row-major [outer, inner] matrix, 128-byte swizzle.
bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_inner,
               uint32_t box_outer, size_t elem_bytes)
{
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * elem_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t es[2] = {1, 1};
    const CUtensorMapDataType dt = elem_bytes == 2   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                     : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const CUresult r = g_encode(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Tile counters of the grouped GEMMs, one per launch of a pass; the pass zeroes
// them on its stream before the first launch.
constexpr int kSchedCounters = 8;

// Offsets of the arrays inside a buffer, laid out in order with 256-byte alignment.
struct Carver {
    size_t off = 0;
    char *base;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <class T> T *take(size_t count)
    {
        off = align_up(off, 256);
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
};

struct Shapes {
    long long T, H, E, I, k, S, G, kk, R, TK;
    long long max_chunks;
    int n_split;              // K splits of the router contraction
};

// Router contraction: one M tile per 128 tokens, K = 3H (three bf16 terms of
// the fp32 router weights).  Split K so that about one wave of 148 SMs is busy;
// the split count divides the number of K blocks.
int router_splits(long long T, long long H)
{
    const long long m_tiles = (T + BM - 1) / BM;
    const long long kb = 3 * H / BK;
    long long target = 148 / m_tiles;
    if (target > kMaxRouterSplits) target = kMaxRouterSplits;
    int best = 1;
    for (int d = 1; d <= target; ++d)
        if (kb % d == 0) best = d;
    return best;
}

Shapes shapes(const moe_cfg &c)
{
    Shapes s;
    s.T = c.T; s.H = c.H; s.E = c.E; s.I = c.I; s.k = c.top_k; s.S = c.n_shared;
    s.G = s.E + s.S;
    s.kk = s.k + s.S;
    s.TK = s.T * s.k;
    s.R = s.TK + s.S * s.T;
    s.max_chunks = (s.TK + kChunkRows - 1) / kChunkRows + s.E;
    s.n_split = router_splits(s.T, s.H);
    return s;
}

// forward state: what the backward reads, plus what the forward needs anyway
struct State {
    int *topk_idx, *counts, *offsets, *gorder, *chunk_start, *perm, *inv_perm, *row_token, *row_slot;
    int *all_rows;
    int *hist;                      // [dispatch chunks, E] per-chunk counts, then base rows
    float *topk_w, *topk_p, *row_w, *rpart;
    __nv_bfloat16 *wr3;
    __nv_bfloat16 *gu, *h, *hw;
    float *O;                       // per-(token, slot) rows: fp32 (BF16), bf16 (MXFP8 forward)
    uint8_t *xq, *xs, *hq, *hs;     // MXFP8 operands
    __nv_bfloat16 *xdq;             // MXFP8 training: the dequantised x (weight-gradient operand)
    int *sched;                     // [kSchedCounters] forward GEMM tile counters
    int *ready;                     // [n_mtiles] per-M-tile readiness (persistent forward)
    int *zero;                      // sched, ready and hist: the counters the persistent forward zeroes
    int n_zero, n_mtiles;
    unsigned long long *gs_flags;   // [kMaxFusedCtas] grid-barrier arrival tags, then release tag, epoch
    size_t bytes;
};

State carve_state(const moe_cfg &c, void *buf, bool training)
{
    const Shapes s = shapes(c);
    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    Carver cv(buf);
    State st{};
    st.topk_idx = cv.take<int>(s.TK);
    st.topk_w = cv.take<float>(s.TK);
    st.topk_p = cv.take<float>(s.TK);
    st.counts = cv.take<int>(s.E);
    st.offsets = cv.take<int>(s.G + 1);
    st.gorder = cv.take<int>(s.G);
    st.chunk_start = cv.take<int>(s.E + 1);
    st.perm = cv.take<int>(s.TK);
    st.inv_perm = cv.take<int>(s.TK);
    st.row_token = cv.take<int>(s.R);
    st.row_slot = cv.take<int>(s.R);
    st.row_w = cv.take<float>(s.R);
    st.all_rows = cv.take<int>(2);
    // tile counters, readiness counters and dispatch histograms in one range, zeroed
    // at the start of the persistent forward (the split forward zeroes the tile
    // counters with a memset; its histograms are written, not accumulated)
    st.n_mtiles = static_cast<int>(s.R / BM + s.G + 1);
    const long long n_hist = ((s.T + kDispatchChunk - 1) / kDispatchChunk) * s.E;
    st.n_zero = static_cast<int>(kSchedCounters + st.n_mtiles + n_hist);
    st.zero = cv.take<int>(st.n_zero);
    st.sched = st.zero;
    st.ready = st.zero + kSchedCounters;
    st.hist = st.ready + st.n_mtiles;
    st.gs_flags = cv.take<unsigned long long>(kMaxFusedCtas + 2);
    st.wr3 = cv.take<__nv_bfloat16>(s.E * 3 * s.H);
    st.rpart = cv.take<float>(static_cast<size_t>(s.n_split) * s.T * 256);
    st.gu = training ? cv.take<__nv_bfloat16>(s.R * 2 * s.I) : nullptr;
    st.hw = training ? cv.take<__nv_bfloat16>(s.R * s.I) : nullptr;
    if (mx) {
        // training also keeps the dequantised h (the down dgrad's slot-gradient operand)
        // and the dequantised x (the gate/up weight gradient's operand)
        st.h = training ? cv.take<__nv_bfloat16>(s.R * s.I) : nullptr;
        st.hq = cv.take<uint8_t>(s.R * s.I);
        st.hs = cv.take<uint8_t>(s.R * s.I / 32);
        st.xq = cv.take<uint8_t>(s.T * s.H);
        st.xs = cv.take<uint8_t>(s.T * s.H / 32);
        st.xdq = training ? cv.take<__nv_bfloat16>(s.T * s.H) : nullptr;
    } else {
        st.h = cv.take<__nv_bfloat16>(s.R * s.I);
        st.hq = st.hs = st.xq = st.xs = nullptr;
        st.xdq = nullptr;
    }
    st.O = mx ? reinterpret_cast<float *>(cv.take<__nv_bfloat16>(s.T * s.kk * s.H)) : cv.take<float>(s.T * s.kk * s.H);
    st.bytes = align_up(cv.off, 256);
    return st;
}

struct BwdScratch {
    float *dl, *partial, *dxs;    // dxs: per-(token, slot) dx rows, fp32
    float *gpart;                 // per routed row and N tile of the down dgrad: <dy W_down, h>
    __nv_bfloat16 *dgu;
    int *sched;                   // [kSchedCounters] backward GEMM tile counters
    int *ready;                   // [n_mtiles] per-M-tile readiness of dGU (persistent backward)
    int *zero;                    // sched and ready: the counters the persistent backward zeroes
    int n_zero;
    unsigned long long *gs_flags; // grid-barrier tags, release tag, epoch
    int *mt_base;                 // [G + 1] first M tile of each group (persistent backward)
    uint8_t *dyq, *dys;           // MXFP8: dy codes [T, H] and scales [T, H/32]
    uint8_t *dguq, *dgus;         // MXFP8: dGU codes [R, 2I] and scales [R, 2I/32]
    size_t bytes;
};

BwdScratch carve_bwd(const moe_cfg &c, void *buf)
{
    const Shapes s = shapes(c);
    Carver cv(buf);
    BwdScratch b{};
    b.dl = cv.take<float>(s.TK);
    b.gpart = cv.take<float>(s.TK * (s.I / 128));
    b.partial = cv.take<float>(s.max_chunks * s.H);
    b.dgu = cv.take<__nv_bfloat16>(s.R * 2 * s.I);
    b.dxs = cv.take<float>(s.T * s.kk * s.H);
    const int n_mtiles = static_cast<int>(s.R / BM + s.G + 1);
    b.n_zero = kSchedCounters + n_mtiles;
    b.zero = cv.take<int>(b.n_zero);
    b.sched = b.zero;
    b.ready = b.zero + kSchedCounters;
    b.gs_flags = cv.take<unsigned long long>(kMaxFusedCtas + 2);
    b.mt_base = cv.take<int>(s.G + 1);
    if (c.dtype == MOK_DTYPE_MXFP8) {
        b.dyq = cv.take<uint8_t>(s.T * s.H);
        b.dys = cv.take<uint8_t>(s.T * s.H / 32);
        b.dguq = cv.take<uint8_t>(s.R * 2 * s.I);
        b.dgus = cv.take<uint8_t>(s.R * 2 * s.I / 32);
    }
    b.bytes = align_up(cv.off, 256);
    return b;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const moe_cfg *c)
{
    if (!c) return MOK_ERR_INVALID;
    if (c->T < 1 || c->H < 256 || c->H % 256 || c->E < 1 || c->E > 256 || c->I < 128 || c->I % 128) return MOK_ERR_INVALID;
    if (c->top_k < 1 || c->top_k > 16 || c->top_k > c->E) return MOK_ERR_INVALID;
    if (c->n_shared < 0 || c->n_shared > 4) return MOK_ERR_INVALID;
    if (c->n_shared > 0 && c->I_shared != c->I) return MOK_ERR_UNSUPPORTED;
    if (c->score_fn != MOK_SCORE_SOFTMAX && c->score_fn != MOK_SCORE_SIGMOID) return MOK_ERR_INVALID;
    if (c->n_group < 1 || c->n_group > 32 || c->E % c->n_group) return MOK_ERR_INVALID;
    if (c->topk_group < 1 || c->topk_group > c->n_group) return MOK_ERR_INVALID;
    if (c->n_group > 1 && c->topk_group < c->n_group && c->top_k > c->topk_group * (c->E / c->n_group))
        return MOK_ERR_INVALID;
    if (!(c->routed_scale > 0.0f)) return MOK_ERR_INVALID;
    if (c->dtype != MOK_DTYPE_BF16 && c->dtype != MOK_DTYPE_MXFP8) return MOK_ERR_INVALID;
    const long long R = (long long)c->T * (c->top_k + c->n_shared);
    if (R >= (1ll << 31)) return MOK_ERR_INVALID;
    return MOK_OK;
}

// One kernel launch on the pass's stream, with the programmatic stream
// serialisation attribute when the pass runs with PDL (the kernels begin with
// griddep_enter, so the attribute only lets a launch's CTAs start early).
template <typename... KArgs, typename... Args>
int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, const char *what,
             Args &&...args)
{
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    if (t_pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
    }
    const cudaError_t e = cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, what, e);
    ++t_launches;
    return MOK_OK;
}

// Operand maps a, b, bs (B of the shared groups) and output maps o, o2, o3.
template <class C>
int launch_wgrad_resident(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &o, const CUtensorMap &o2,
                          const GemmArgs &args, int grid, cudaStream_t st)
{
    if (grid <= 0) return MOK_OK;
    cudaError_t e = cudaFuncSetAttribute(wgrad_resident_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(wgrad_resident_kernel)", e);
    return launch_k(wgrad_resident_kernel<C>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st,
                    "wgrad_resident_kernel launch", a, b, o, o2, args);
}

// M tiles per resident work unit: runs of at most 16, split evenly
int resident_m_per_unit(int m_tiles)
{
    const int chunks = (m_tiles + 15) / 16;
    return (m_tiles + chunks - 1) / chunks;
}

template <class C>
int launch_gemm(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &bs, const CUtensorMap &o,
                const CUtensorMap &o2, const CUtensorMap &o3, const GemmArgs &args, int grid, cudaStream_t st)
{
    if (grid <= 0) return MOK_OK;
    if (!args.sched) return fail(MOK_ERR_INVALID, "grouped GEMM launch without a tile counter");
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(grouped_gemm_kernel)", e);
    return launch_k(grouped_gemm_kernel<C>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st,
                    "grouped_gemm_kernel launch", a, b, bs, o, o2, o3, args);
}

inline int blocks_for(long long n, int per) { return static_cast<int>((n + per - 1) / per); }

#define MOK_TRY(expr)                 \
    do {                              \
        const int rc_ = (expr);       \
        if (rc_ != MOK_OK) return rc_; \
    } while (0)

#define MOK_LAUNCHED()                                                              \
    do {                                                                            \
        const cudaError_t e_ = cudaGetLastError();                                  \
        if (e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "kernel launch", e_);    \
        ++t_launches;                                                               \
    } while (0)

// ------------------------------------------------------------------ forward
// Tensor maps and arguments of every step of the forward, shared by the split
// schedule (one launch per step) and the persistent one (one launch).
struct FwdPlan {
    FusedMaps m;
    GemmArgs gr, ga, gd;
    SelectArgs sa;
    DispatchArgs da;
    int n_chunks;
};

// Router logits, top-k and dispatch of the forward (every schedule, and the
// routing phase of expert parallelism).
int build_route_plan(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const DeviceInfo &dev,
                     FwdPlan &pl)
{
    const Shapes s = shapes(c);
    // router logits on the tensor cores: x . [Wr_hi | Wr_mid | Wr_lo]^T, split over K
    if (!make_tmap(&pl.m.rA, x, s.H, s.T, BK, 128, 2)) return fail(MOK_ERR_INVALID, "tensor map (x)");
    if (!make_tmap(&pl.m.rB, st.wr3, 3 * s.H, s.E, BK, 256, 2)) return fail(MOK_ERR_INVALID, "tensor map (router)");
    if (!make_tmap(&pl.m.rO, st.rpart, 256, s.n_split * s.T, 32, 32, 4)) return fail(MOK_ERR_INVALID, "tensor map (logits)");
    GemmArgs &gr = pl.gr;
    gr = GemmArgs{};
    gr.num_groups = 1;
    gr.num_routed = 1;
    gr.offsets = st.all_rows;
    gr.n_tiles = s.n_split;
    gr.num_kb = static_cast<int>(3 * s.H / BK / s.n_split);
    gr.a_k_mod = c.H;
    gr.out_f32 = st.rpart;
    gr.rows_total = c.T;
    gr.status = dev.status;
    gr.sched = st.sched + 0;

    SelectArgs &sa = pl.sa;
    sa.partial = st.rpart;
    sa.n_split = s.n_split;
    sa.e_bias = p.e_bias;
    sa.logit_bias = p.logit_bias;
    sa.T = c.T; sa.E = c.E; sa.k = c.top_k;
    sa.score_fn = c.score_fn; sa.n_group = c.n_group; sa.topk_group = c.topk_group;
    sa.routed_scale = c.routed_scale;
    sa.topk_idx = st.topk_idx; sa.topk_w = st.topk_w; sa.topk_p = st.topk_p;
    sa.hist = nullptr;

    DispatchArgs &da = pl.da;
    da.topk_idx = st.topk_idx; da.topk_w = st.topk_w;
    da.T = c.T; da.k = c.top_k; da.E = c.E; da.S = c.n_shared; da.chunk_rows = kChunkRows;
    da.counts = st.counts; da.offsets = st.offsets; da.gorder = st.gorder; da.chunk_start = st.chunk_start;
    da.perm = st.perm; da.inv_perm = st.inv_perm; da.row_token = st.row_token; da.row_slot = st.row_slot;
    da.row_w = st.row_w;
    da.hist = st.hist;
    da.status = dev.status;
    pl.n_chunks = static_cast<int>((s.T + kDispatchChunk - 1) / kDispatchChunk);
    return MOK_OK;
}

int build_fwd_plan(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const DeviceInfo &dev,
                   bool training, FwdPlan &pl)
{
    const Shapes s = shapes(c);
    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    MOK_TRY(build_route_plan(c, x, p, st, dev, pl));

    GemmArgs &ga = pl.ga;
    GemmArgs &gd = pl.gd;
    ga = GemmArgs{};
    ga.sched = st.sched + 1;
    ga.num_groups = static_cast<int>(s.G);
    ga.num_routed = c.E;
    ga.offsets = st.offsets;
    ga.row_token = st.row_token;
    ga.row_slot = st.row_slot;
    ga.row_w = st.row_w;
    ga.n_tiles = c.I / 128;
    ga.b_rows_per_group = 2 * c.I;
    ga.b_half = c.I;
    ga.inter = c.I;
    ga.gather_ld = c.H;
    ga.status = dev.status;
    ga.test_drop_signal = t_drop_signal;
    ga.ready = st.ready;
    if (mx) {
        // MXFP8: block-scaled expert GEMMs on the quantised x (1x32 ue8m0 blocks along H)
        if (!make_tmap(&pl.m.gB, p.w_gate_up, s.H, s.E * 2 * s.I, 128, 128, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gBs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : s.E) * 2 * s.I, 128, 128, 1))
            return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gO, st.hq, s.I, s.R, 128, 32, 1)) return MOK_ERR_INVALID;
        pl.m.gO2 = pl.m.gO3 = pl.m.gO;
        ga.num_kb = c.H / 128;
        ga.out = reinterpret_cast<__nv_bfloat16 *>(st.hq);
        ga.out_scales = st.hs;
        ga.out2 = training ? st.gu : nullptr;       // training: g/u, the dequantised h, w * h
        ga.out_hb = training ? st.h : nullptr;
        ga.out3 = training ? st.hw : nullptr;
        ga.gather_src = reinterpret_cast<const __nv_bfloat16 *>(st.xq);
        ga.sfa_src = st.xs;
        ga.sfb_src = p.s_gate_up;
        ga.sfb_src_s = s.S ? p.ss_gate_up : p.s_gate_up;
        ga.sf_ld = c.H / 32;
        ga.sfb_row_tiles = static_cast<int>(s.E * 2 * s.I / 128);
        ga.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : s.E) * 2 * s.I / 128);

        if (!make_tmap(&pl.m.dA, st.hq, s.I, s.R, 128, 128, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dB, p.w_down, s.I, s.E * s.H, 128, 256, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dBs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : s.E) * s.H, 128, 256, 1))
            return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dO, st.O, s.H, s.T * s.kk, 64, 1, 2)) return MOK_ERR_INVALID;   // bf16 slot rows
        gd = ga;
        gd.sched = st.sched + 2;
        gd.n_tiles = c.H / 256;
        gd.num_kb = c.I / 128;
        gd.b_rows_per_group = c.H;
        gd.b_half = 0;
        gd.out = reinterpret_cast<__nv_bfloat16 *>(st.O);
        gd.out_f32 = nullptr;
        gd.out_scales = nullptr;
        gd.out2 = gd.out3 = gd.out_hb = nullptr;
        gd.ldo = c.H;
        gd.gather_src = nullptr;
        gd.sfa_src = st.hs;
        gd.sfb_src = p.s_down;
        gd.sfb_src_s = s.S ? p.ss_down : p.s_down;
        gd.sf_ld = c.I / 32;
        gd.sfb_row_tiles = static_cast<int>(s.E * s.H / 128);
        gd.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : s.E) * s.H / 128);
    } else {
        // gate/up: pull token rows by index, SwiGLU epilogue
        if (!make_tmap(&pl.m.gB, p.w_gate_up, s.H, s.E * 2 * s.I, BK, 128, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gO, st.h, s.I, s.R, 64, 32, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gO2, training ? st.gu : st.h, training ? 2 * s.I : s.I, s.R, 64, 32, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gO3, training ? st.hw : st.h, s.I, s.R, 64, 32, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.gBs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : s.E) * 2 * s.I, BK, 128, 2))
            return MOK_ERR_INVALID;
        ga.num_kb = c.H / BK;
        ga.out = st.h;
        ga.out2 = training ? st.gu : nullptr;
        ga.out3 = training ? st.hw : nullptr;
        ga.gather_src = static_cast<const __nv_bfloat16 *>(x);

        // down: contiguous h rows, push epilogue into (token, slot) rows
        if (!make_tmap(&pl.m.dA, st.h, s.I, s.R, BK, 128, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dB, p.w_down, s.I, s.E * s.H, BK, 256, 2)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dBs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : s.E) * s.H, BK, 256, 2))
            return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.dO, st.O, s.H, s.T * s.kk, 32, 1, 4)) return MOK_ERR_INVALID;
        gd = ga;
        gd.sched = st.sched + 2;
        gd.n_tiles = c.H / 256;
        gd.num_kb = c.I / BK;
        gd.b_rows_per_group = c.H;
        gd.b_half = 0;
        gd.out = nullptr;
        gd.out_f32 = st.O;
        gd.out2 = gd.out3 = nullptr;
        gd.ldo = c.H;
    }
    gd.ready_target = 4 * (c.I / 128);    // four epilogue warps per gate/up tile, I/128 tiles per M tile
    return MOK_OK;
}

int copy_routing(const moe_routing *routing, const State &st, const Shapes &s, cudaStream_t stream)
{
    if (!routing) return MOK_OK;
    const size_t tk = static_cast<size_t>(s.TK);
    struct { void *dst; const void *src; size_t n; } cp[] = {
        {routing->topk_idx, st.topk_idx, tk * 4}, {routing->topk_w, st.topk_w, tk * 4},
        {routing->counts, st.counts, static_cast<size_t>(s.E) * 4},
        {routing->offsets, st.offsets, static_cast<size_t>(s.E + 1) * 4},
        {routing->perm, st.perm, tk * 4}, {routing->inv_perm, st.inv_perm, tk * 4}};
    for (const auto &q : cp)
        if (q.dst)
            if (const cudaError_t e = cudaMemcpyAsync(q.dst, q.src, q.n, cudaMemcpyDeviceToDevice, stream); e != cudaSuccess)
                return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync(routing)", e);
    return MOK_OK;
}

// Router split, router GEMM and top-k (the split schedule's first launches).
int launch_router(const moe_cfg &c, const moe_params &p, const State &st, const DeviceInfo &dev, const FwdPlan &pl,
                  cudaStream_t stream)
{
    const Shapes s = shapes(c);
    MOK_TRY(launch_k(router_split_kernel, dim3(blocks_for(s.E * s.H, 256)), dim3(256), 0, stream, "router_split_kernel",
                     p.router_w, st.wr3, c.E, c.H, st.all_rows, c.T));
    MOK_TRY(launch_gemm<typename FusedCfg<false>::Router>(pl.m.rA, pl.m.rB, pl.m.rB, pl.m.rO, pl.m.rO, pl.m.rO, pl.gr,
                                                         dev.sms, stream));
    return launch_k(router_select_kernel, dim3(blocks_for(s.T, 8)), dim3(256), 0, stream, "router_select_kernel", pl.sa);
}

// Counts, scan and placement of the sorted rows.
int launch_dispatch(const FwdPlan &pl, cudaStream_t stream)
{
    MOK_TRY(launch_k(dispatch_count_kernel, dim3(pl.n_chunks), dim3(kDispatchChunk), 0, stream, "dispatch_count_kernel",
                     pl.da));
    MOK_TRY(launch_k(dispatch_scan_kernel, dim3(1), dim3(256), 0, stream, "dispatch_scan_kernel", pl.da, pl.n_chunks));
    return launch_k(dispatch_place_kernel, dim3(pl.n_chunks), dim3(kDispatchChunk), 0, stream, "dispatch_place_kernel",
                    pl.da);
}

// Split schedule: one launch per step, in stream order.
int forward_split(const moe_cfg &c, const void *x, const moe_params &p, void *y, const State &st,
                  const DeviceInfo &dev, const FwdPlan &pl, cudaStream_t stream)
{
    const Shapes s = shapes(c);
    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    if (const cudaError_t e = cudaMemsetAsync(st.sched, 0, kSchedCounters * sizeof(int), stream); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaMemsetAsync(tile counters)", e);
    MOK_TRY(mark_fwd(0, stream));
    MOK_TRY(launch_router(c, p, st, dev, pl, stream));
    MOK_TRY(mark_fwd(1, stream));
    MOK_TRY(launch_dispatch(pl, stream));

    MOK_TRY(mark_fwd(2, stream));
    GemmArgs ga = pl.ga, gd = pl.gd;
    ga.ready_role = gd.ready_role = kReadyNone;
    if (mx) {
        const long long xb = s.T * s.H / 32;
        MOK_TRY(launch_k(quantize_mxfp8_kernel, dim3(blocks_for(xb, 256)), dim3(256), 0, stream, "quantize_mxfp8_kernel",
                         static_cast<const __nv_bfloat16 *>(x), xb, st.xq, st.xs, static_cast<long long>(s.H / 32), 0ll,
                         st.xdq));
        MOK_TRY(launch_gemm<typename FusedCfg<true>::GateUp>(pl.m.gB, pl.m.gB, pl.m.gBs, pl.m.gO, pl.m.gO2, pl.m.gO3,
                                                            ga, dev.sms, stream));
        MOK_TRY(mark_fwd(3, stream));
        MOK_TRY(launch_gemm<typename FusedCfg<true>::Down>(pl.m.dA, pl.m.dB, pl.m.dBs, pl.m.dO, pl.m.dO, pl.m.dO, gd,
                                                          dev.sms, stream));
    } else {
        MOK_TRY(launch_gemm<typename FusedCfg<false>::GateUp>(pl.m.gB, pl.m.gB, pl.m.gBs, pl.m.gO, pl.m.gO2, pl.m.gO3,
                                                             ga, dev.sms, stream));
        MOK_TRY(mark_fwd(3, stream));
        MOK_TRY(launch_gemm<typename FusedCfg<false>::Down>(pl.m.dA, pl.m.dB, pl.m.dBs, pl.m.dO, pl.m.dO, pl.m.dO, gd,
                                                           dev.sms, stream));
    }

    MOK_TRY(mark_fwd(4, stream));
    if (mx)
        MOK_TRY(launch_k(combine_kernel<__nv_bfloat16>, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0, stream,
                         "combine_kernel", reinterpret_cast<const __nv_bfloat16 *>(st.O),
                         static_cast<const float *>(st.topk_w), static_cast<__nv_bfloat16 *>(y), c.T, c.H, c.top_k,
                         c.n_shared));
    else
        MOK_TRY(launch_k(combine_kernel<float>, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0, stream,
                         "combine_kernel", static_cast<const float *>(st.O), static_cast<const float *>(st.topk_w),
                         static_cast<__nv_bfloat16 *>(y), c.T, c.H, c.top_k, c.n_shared));
    return mark_fwd(5, stream);
}

// Persistent schedule: the whole forward as one cooperative launch (fused.cuh).
// Cooperative, so that every CTA is resident at once (the grid barriers and the
// readiness waits need that) or the launch fails; one CTA per SM.
template <bool MX>
int launch_fused(const moe_cfg &c, const void *x, const moe_params &p, void *y, const State &st,
                 const DeviceInfo &dev, const FwdPlan &pl, cudaStream_t stream)
{
    using F = FusedCfg<MX>;
    if (dev.sms > kMaxFusedCtas) return fail(MOK_ERR_UNSUPPORTED, "more SMs than the grid barrier holds");
    FusedFwdArgs a{};
    a.gs.flags = st.gs_flags;
    a.gs.go = st.gs_flags + kMaxFusedCtas;
    a.gs.epoch = st.gs_flags + kMaxFusedCtas + 1;
    a.status = dev.status;
    a.zero = st.zero;
    a.n_zero = st.n_zero;
    a.router_w = p.router_w;
    a.wr3 = st.wr3;
    a.all_rows = st.all_rows;
    a.T = c.T; a.H = c.H; a.E = c.E; a.k = c.top_k; a.S = c.n_shared;
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.xq = st.xq;
    a.xs = st.xs;
    a.xdq = st.xdq;
    a.gr = pl.gr;
    a.ga = pl.ga;
    a.gd = pl.gd;
    a.ga.ready_role = kReadySignal;
    a.gd.ready_role = kReadyWait;
    a.sa = pl.sa;
    a.sa.hist = st.hist;
    a.da = pl.da;
    a.n_chunks = pl.n_chunks;
    a.O = st.O;
    a.y = static_cast<__nv_bfloat16 *>(y);
    a.trace = (t_dev_trace && t_dev_trace_bytes >= sizeof(unsigned long long) * kFusedTracePoints * dev.sms)
                  ? t_dev_trace : nullptr;

    cudaError_t e = cudaFuncSetAttribute(moe_fwd_fused_kernel<MX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         F::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(moe_fwd_fused_kernel)", e);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(dev.sms));
    lc.blockDim = dim3(kFusedThreads);
    lc.dynamicSmemBytes = F::SMEM_BYTES;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    MOK_TRY(mark_fwd(0, stream));
    e = cudaLaunchKernelEx(&lc, moe_fwd_fused_kernel<MX>, pl.m, a);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaLaunchKernelEx(moe_fwd_fused_kernel, cooperative)", e);
    ++t_launches;
    // one launch: the per-step events all mark its end (phase times come from moe_trace_device)
    for (int i = 1; i <= MOK_FWD_PHASES; ++i) MOK_TRY(mark_fwd(i, stream));
    return MOK_OK;
}

int forward(const moe_cfg &c, const void *x, const moe_params &p, void *y, const moe_routing *routing,
            const State &st, const DeviceInfo &dev, bool training, cudaStream_t stream)
{
    t_launches = 0;
    FwdPlan pl;
    MOK_TRY(build_fwd_plan(c, x, p, st, dev, training, pl));
    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    t_pdl = t_schedule == MOK_SCHEDULE_SPLIT_PDL;
    if (t_schedule == MOK_SCHEDULE_SPLIT || t_schedule == MOK_SCHEDULE_SPLIT_PDL) {
        MOK_TRY(forward_split(c, x, p, y, st, dev, pl, stream));
    } else if (mx) {
        MOK_TRY(launch_fused<true>(c, x, p, y, st, dev, pl, stream));
    } else {
        MOK_TRY(launch_fused<false>(c, x, p, y, st, dev, pl, stream));
    }
    return copy_routing(routing, st, shapes(c), stream);
}

// ------------------------------------------------------------------ backward
// Tensor maps and arguments of every step of the backward, shared by the split
// schedule and the persistent one.
struct BwdPlan {
    FusedBwdMaps m;
    GemmArgs g1, g2, g3, g4;
    bool mx;                    // MXFP8 data gradients
    const void *dy;             // [T, H] bf16 (quantised first under MXFP8)
    int g2_grid, g4_grid;       // split launches of the streaming weight gradients
    int g2_units, g4_units;     // resident weight-gradient work units (0: none)
    bool n256;                  // I is a multiple of 256
};

int build_bwd_plan(const moe_cfg &c, const void *x, const void *dy, const moe_params &p, const State &st,
                   const moe_grads &gr, const BwdScratch &bs, const DeviceInfo &dev, BwdPlan &pl)
{
    const Shapes s = shapes(c);
    pl.n256 = c.I % 256 == 0;
    pl.dy = dy;
    GemmArgs base{};
    base.num_groups = static_cast<int>(s.G);
    base.num_routed = c.E;
    base.offsets = st.offsets;
    base.gorder = st.gorder;
    base.row_token = st.row_token;
    base.row_slot = st.row_slot;
    base.row_w = st.row_w;
    base.inter = c.I;
    base.gather_src = static_cast<const __nv_bfloat16 *>(dy);
    base.gather_ld = c.H;
    base.status = dev.status;
    base.ready = bs.ready;

    // dgrad of down: dh = w * (dy[token] . W_down), SwiGLU backward epilogue -> dGU
    if (!make_tmap(&pl.m.d1B, p.w_down, s.I, s.E * s.H, 64, 64, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.d1Bs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : s.E) * s.H, 64, 64, 2))
        return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.d1O, bs.dgu, 2 * s.I, s.R, 64, 32, 2)) return MOK_ERR_INVALID;
    GemmArgs &g1 = pl.g1;
    g1 = base;
    g1.sched = bs.sched + 0;
    g1.num_kb = c.H / BK;
    g1.b_rows_per_group = c.H;
    g1.aux = st.gu;
    g1.aux_h = st.h;
    g1.gpart = bs.gpart;
    g1.out = bs.dgu;
    g1.n_tiles = pl.n256 ? c.I / 256 : c.I / 128;   // N = 256 halves the gathered dy rows per weight byte
    g1.test_drop_signal = t_drop_signal;

    // wgrad of down: dW_down[g] = sum_r dy[token r]^T (w_r h_r)
    if (!make_tmap(&pl.m.w2O, gr.dw_down, s.I, s.E * s.H, 64, 32, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.w2O2, s.S ? gr.dws_down : gr.dw_down, s.I, (s.S ? s.S : s.E) * s.H, 64, 32, 2))
        return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.w2B, st.hw, s.I, s.R, 64, 64, 2)) return MOK_ERR_INVALID;
    GemmArgs &g2 = pl.g2;
    g2 = base;
    g2.sched = bs.sched + 1;
    g2.m_tiles = c.H / 128;
    g2.out = static_cast<__nv_bfloat16 *>(gr.dw_down);
    g2.out_s = static_cast<__nv_bfloat16 *>(gr.dws_down);
    g2.ldo = c.I;
    g2.group_out_elems = s.H * s.I;
    if (pl.n256) {
        // groups of more than kResidentRows rows stream both operands; the rest keep
        // their (w h) slab resident and stream gathered dy
        g2.n_tiles = c.I / 256;
        g2.k_split = kResidentRows;
        g2.m_per_unit = resident_m_per_unit(g2.m_tiles);
        pl.g2_units = static_cast<int>(s.G * g2.n_tiles * ((g2.m_tiles + g2.m_per_unit - 1) / g2.m_per_unit));
    } else {
        g2.n_tiles = c.I / 128;
        pl.g2_units = 0;
    }
    const long long t2 = s.G * g2.m_tiles * g2.n_tiles;
    pl.g2_grid = static_cast<int>(t2 < dev.sms ? t2 : dev.sms);

    // dgrad of gate/up: dX rows = dGU . W_gate_up, pushed into (token, slot) rows
    if (!make_tmap(&pl.m.d3A, bs.dgu, 2 * s.I, s.R, BK, 128, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.d3B, p.w_gate_up, s.H, s.E * 2 * s.I, 64, 64, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.d3Bs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : s.E) * 2 * s.I, 64, 64, 2))
        return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.d3O, bs.dxs, s.H, s.T * s.kk, 32, 1, 4)) return MOK_ERR_INVALID;
    GemmArgs &g3 = pl.g3;
    g3 = base;
    g3.sched = bs.sched + 2;
    g3.n_tiles = c.H / 256;
    g3.num_kb = 2 * c.I / BK;
    g3.b_rows_per_group = 2 * c.I;
    g3.out_f32 = bs.dxs;
    g3.ldo = c.H;
    g3.ready_target = 4 * g1.n_tiles;     // four epilogue warps per down-dgrad tile, its N tiles per M tile

    pl.mx = c.dtype == MOK_DTYPE_MXFP8;
    if (pl.mx) {
        // down dgrad on MXFP8 operands: dy codes (gathered by token) x W_down^T (K = H)
        if (!make_tmap(&pl.m.d1B, p.wt_down, s.H, s.E * s.I, 128, 256, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.d1Bs, s.S ? p.wst_down : p.wt_down, s.H, (s.S ? s.S : s.E) * s.I, 128, 256, 1))
            return MOK_ERR_INVALID;
        g1.num_kb = c.H / 128;
        g1.b_rows_per_group = c.I;
        g1.n_tiles = c.I / 256;
        g1.gather_src = reinterpret_cast<const __nv_bfloat16 *>(bs.dyq);
        g1.sfa_src = bs.dys;
        g1.sf_ld = c.H / 32;
        g1.sfb_src = p.st_down;
        g1.sfb_src_s = s.S ? p.sst_down : p.st_down;
        g1.sfb_row_tiles = static_cast<int>(s.E * s.I / 128);
        g1.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : s.E) * s.I / 128);
        g1.out_q = bs.dguq;
        g1.out_scales = bs.dgus;
        // gate/up dgrad on MXFP8 operands: dGU codes x W_gate_up^T (K = 2I)
        if (!make_tmap(&pl.m.d3A, bs.dguq, 2 * s.I, s.R, 128, 128, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.d3B, p.wt_gate_up, 2 * s.I, s.E * s.H, 128, 256, 1)) return MOK_ERR_INVALID;
        if (!make_tmap(&pl.m.d3Bs, s.S ? p.wst_gate_up : p.wt_gate_up, 2 * s.I, (s.S ? s.S : s.E) * s.H, 128, 256, 1))
            return MOK_ERR_INVALID;
        g3.num_kb = 2 * c.I / 128;
        g3.b_rows_per_group = c.H;
        g3.gather_src = nullptr;
        g3.sfa_src = bs.dgus;
        g3.sf_ld = 2 * c.I / 32;
        g3.sfb_src = p.st_gate_up;
        g3.sfb_src_s = s.S ? p.sst_gate_up : p.st_gate_up;
        g3.sfb_row_tiles = static_cast<int>(s.E * s.H / 128);
        g3.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : s.E) * s.H / 128);
    }

    // wgrad of gate/up: dW_gate_up[g] = sum_r dGU_r^T x[token r]
    if (!make_tmap(&pl.m.w4A, bs.dgu, 2 * s.I, s.R, 64, 64, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.w4O, gr.dw_gate_up, s.H, s.E * 2 * s.I, 64, 32, 2)) return MOK_ERR_INVALID;
    if (!make_tmap(&pl.m.w4O2, s.S ? gr.dws_gate_up : gr.dw_gate_up, s.H, (s.S ? s.S : s.E) * 2 * s.I, 64, 32, 2))
        return MOK_ERR_INVALID;
    GemmArgs &g4 = pl.g4;
    g4 = base;
    g4.sched = bs.sched + 3;
    g4.gather_src = pl.mx ? st.xdq : static_cast<const __nv_bfloat16 *>(x);   // MXFP8: the x the forward used
    g4.m_tiles = 2 * c.I / 128;
    g4.n_tiles = c.H / 256;
    g4.out = static_cast<__nv_bfloat16 *>(gr.dw_gate_up);
    g4.out_s = static_cast<__nv_bfloat16 *>(gr.dws_gate_up);
    g4.ldo = c.H;
    g4.group_out_elems = 2 * s.I * s.H;
    g4.k_split = kResidentRows;            // larger groups stream; the rest keep their x slab resident
    g4.m_per_unit = resident_m_per_unit(g4.m_tiles);
    const long long t4 = s.G * g4.m_tiles * g4.n_tiles;
    pl.g4_grid = static_cast<int>(t4 < dev.sms ? t4 : dev.sms);
    pl.g4_units = static_cast<int>(s.G * g4.n_tiles * ((g4.m_tiles + g4.m_per_unit - 1) / g4.m_per_unit));
    return MOK_OK;
}

// Split schedule: one launch per step, in stream order (with PDL unless the plain
// split schedule is asked for).
int backward_split(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const moe_grads &gr,
                   const BwdScratch &bs, const DeviceInfo &dev, const BwdPlan &pl, cudaStream_t stream)
{
    const Shapes s = shapes(c);
    t_pdl = t_schedule != MOK_SCHEDULE_SPLIT;
    if (const cudaError_t e = cudaMemsetAsync(bs.sched, 0, kSchedCounters * sizeof(int), stream); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaMemsetAsync(tile counters)", e);
    GemmArgs g1 = pl.g1, g2 = pl.g2, g3 = pl.g3, g4 = pl.g4;
    g1.ready_role = g3.ready_role = kReadyNone;
    const FusedBwdMaps &m = pl.m;

    MOK_TRY(mark_bwd(0, stream));
    if (pl.mx) {
        const long long nb = s.T * s.H / 32;
        MOK_TRY(launch_k(quantize_mxfp8_kernel, dim3(blocks_for(nb, 256)), dim3(256), 0, stream, "quantize_mxfp8_kernel",
                         static_cast<const __nv_bfloat16 *>(pl.dy), nb, bs.dyq, bs.dys,
                         static_cast<long long>(s.H / 32), 0ll, static_cast<__nv_bfloat16 *>(nullptr)));
        MOK_TRY(launch_gemm<DgradDownMX>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1, dev.sms, stream));
    } else if (pl.n256)
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::DgradDown>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1,
                                                                  dev.sms, stream));
    else
        MOK_TRY(launch_gemm<typename FusedBwdCfg<false>::DgradDown>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1,
                                                                   dev.sms, stream));

    // slot gradients from the down dgrad's partials, then the router weight gradient
    MOK_TRY(mark_bwd(1, stream));
    MOK_TRY(launch_k(slot_grad_kernel, dim3(blocks_for(s.T, 256)), dim3(256), 0, stream, "slot_grad_kernel",
                     static_cast<const float *>(bs.gpart), g1.n_tiles, static_cast<const int *>(st.inv_perm),
                     static_cast<const float *>(st.topk_w), static_cast<const float *>(st.topk_p), bs.dl, c.T,
                     c.top_k, c.score_fn, c.routed_scale));
    MOK_TRY(mark_bwd(2, stream));
    MOK_TRY(launch_k(drouter_partial_kernel, dim3(static_cast<unsigned>(s.max_chunks), c.H / 256), dim3(256), 0, stream,
                     "drouter_partial_kernel", static_cast<const __nv_bfloat16 *>(x), static_cast<const float *>(bs.dl),
                     static_cast<const int *>(st.offsets), static_cast<const int *>(st.chunk_start),
                     static_cast<const int *>(st.perm), bs.partial, c.H, c.E, c.top_k, kChunkRows));
    MOK_TRY(mark_bwd(3, stream));
    MOK_TRY(launch_k(drouter_reduce_kernel, dim3(blocks_for(s.E * s.H, 256)), dim3(256), 0, stream,
                     "drouter_reduce_kernel", static_cast<const float *>(bs.partial),
                     static_cast<const int *>(st.chunk_start), gr.drouter_w, c.H, c.E));

    MOK_TRY(mark_bwd(4, stream));
    if (pl.n256) {
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::WgradDown>(m.w2B, m.w2B, m.w2B, m.w2O, m.w2O2, m.w2O, g2,
                                                                  pl.g2_grid, stream));
        MOK_TRY(launch_wgrad_resident<WgradResCfg<true>>(m.w2B, m.w2B, m.w2O, m.w2O2, g2,
                                                         pl.g2_units < dev.sms ? pl.g2_units : dev.sms, stream));
    } else {
        MOK_TRY(launch_gemm<typename FusedBwdCfg<false>::WgradDown>(m.w2B, m.w2B, m.w2B, m.w2O, m.w2O2, m.w2O, g2,
                                                                   pl.g2_grid, stream));
    }

    MOK_TRY(mark_bwd(5, stream));
    if (pl.mx)
        MOK_TRY(launch_gemm<DgradGUMX>(m.d3A, m.d3B, m.d3Bs, m.d3O, m.d3O, m.d3O, g3, dev.sms, stream));
    else
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::DgradGU>(m.d3A, m.d3B, m.d3Bs, m.d3O, m.d3O, m.d3O, g3,
                                                                dev.sms, stream));

    MOK_TRY(mark_bwd(6, stream));
    MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::WgradGU>(m.w4A, m.w4A, m.w4A, m.w4O, m.w4O2, m.w4O, g4, pl.g4_grid,
                                                            stream));
    MOK_TRY(launch_wgrad_resident<WgradResCfg<false>>(m.w4A, m.w4A, m.w4O, m.w4O2, g4,
                                                      pl.g4_units < dev.sms ? pl.g4_units : dev.sms, stream));

    MOK_TRY(mark_bwd(7, stream));
    MOK_TRY(launch_k(dx_combine_kernel, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0, stream,
                     "dx_combine_kernel", static_cast<const float *>(bs.dxs), static_cast<const float *>(bs.dl),
                     static_cast<const int *>(st.topk_idx), p.router_w, static_cast<__nv_bfloat16 *>(gr.dx), c.T, c.H,
                     c.top_k, c.n_shared));
    return mark_bwd(8, stream);
}

// Persistent schedule: the whole backward as one cooperative launch (fused_bwd.cuh).
template <bool N256, bool MX>
int launch_fused_bwd(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const moe_grads &gr,
                     const BwdScratch &bs, const DeviceInfo &dev, const BwdPlan &pl, cudaStream_t stream)
{
    using F = FusedBwdCfg<N256, MX>;
    if (dev.sms > kMaxFusedCtas) return fail(MOK_ERR_UNSUPPORTED, "more SMs than the grid barrier holds");
    const Shapes s = shapes(c);
    FusedBwdArgs a{};
    a.gs.flags = bs.gs_flags;
    a.gs.go = bs.gs_flags + kMaxFusedCtas;
    a.gs.epoch = bs.gs_flags + kMaxFusedCtas + 1;
    a.status = dev.status;
    a.zero = bs.zero;
    a.n_zero = bs.n_zero;
    a.g1 = pl.g1;
    a.g1.ready_role = kReadySignal;
    a.g2 = a.g2r = pl.g2;
    a.g3 = pl.g3;
    a.g3.ready_role = kReadyWait;
    a.g4 = a.g4r = pl.g4;
    a.g4.ready_role = a.g4r.ready_role = kReadyWaitGroup;
    a.g4.ready_target = a.g4r.ready_target = 4 * pl.g1.n_tiles;
    a.g4.mt_base = a.g4r.mt_base = bs.mt_base;
    a.offsets_all = st.offsets;
    a.mt_base = bs.mt_base;
    a.g2_units = pl.g2_units;
    a.g4_units = pl.g4_units;
    a.gpart = bs.gpart;
    a.n_parts = pl.g1.n_tiles;
    a.inv_perm = st.inv_perm;
    a.topk_idx = st.topk_idx;
    a.offsets = st.offsets;
    a.chunk_start = st.chunk_start;
    a.perm = st.perm;
    a.topk_w = st.topk_w;
    a.topk_p = st.topk_p;
    a.router_w = p.router_w;
    a.dl = bs.dl;
    a.partial = bs.partial;
    a.drouter_w = gr.drouter_w;
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.T = c.T; a.H = c.H; a.E = c.E; a.k = c.top_k; a.S = c.n_shared;
    a.score_fn = c.score_fn;
    a.chunk_rows = kChunkRows;
    a.max_chunks = static_cast<int>(s.max_chunks);
    a.routed_scale = c.routed_scale;
    a.dxs = bs.dxs;
    a.dx = static_cast<__nv_bfloat16 *>(gr.dx);
    a.dy = static_cast<const __nv_bfloat16 *>(pl.dy);
    a.dyq = bs.dyq;
    a.dys = bs.dys;
    a.trace = (t_dev_trace_bwd && t_dev_trace_bwd_bytes >= sizeof(unsigned long long) * kFusedBwdTracePoints * dev.sms)
                  ? t_dev_trace_bwd : nullptr;

    cudaError_t e = cudaFuncSetAttribute(moe_bwd_fused_kernel<N256, MX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         F::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(moe_bwd_fused_kernel)", e);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(dev.sms));
    lc.blockDim = dim3(kFusedThreads);
    lc.dynamicSmemBytes = F::SMEM_BYTES;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    MOK_TRY(mark_bwd(0, stream));
    e = cudaLaunchKernelEx(&lc, moe_bwd_fused_kernel<N256, MX>, pl.m, a);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaLaunchKernelEx(moe_bwd_fused_kernel, cooperative)", e);
    ++t_launches;
    for (int i = 1; i <= MOK_BWD_PHASES; ++i) MOK_TRY(mark_bwd(i, stream));
    return MOK_OK;
}

int backward(const moe_cfg &c, const void *x, const void *dy, const moe_params &p, const State &st,
             const moe_grads &gr, const BwdScratch &bs, const DeviceInfo &dev, cudaStream_t stream)
{
    t_launches = 0;
    BwdPlan pl;
    MOK_TRY(build_bwd_plan(c, x, dy, p, st, gr, bs, dev, pl));
    if (t_schedule == MOK_SCHEDULE_PERSISTENT) {
        t_pdl = false;
        if (pl.mx) return launch_fused_bwd<true, true>(c, x, p, st, gr, bs, dev, pl, stream);
        return pl.n256 ? launch_fused_bwd<true, false>(c, x, p, st, gr, bs, dev, pl, stream)
                       : launch_fused_bwd<false, false>(c, x, p, st, gr, bs, dev, pl, stream);
    }
    return backward_split(c, x, p, st, gr, bs, dev, pl, stream);
}

int check_params(const moe_cfg &c, const moe_params *p)
{
    if (!p || !p->router_w || !p->w_gate_up || !p->w_down) return MOK_ERR_INVALID;
    if (c.n_shared > 0 && (!p->ws_gate_up || !p->ws_down)) return MOK_ERR_INVALID;
    if (c.dtype == MOK_DTYPE_MXFP8 && (!p->s_gate_up || !p->s_down || (c.n_shared > 0 && (!p->ss_gate_up || !p->ss_down))))
        return MOK_ERR_INVALID;
    const void *ptrs[] = {p->router_w, p->w_gate_up, p->w_down, p->ws_gate_up, p->ws_down};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return MOK_ERR_INVALID;
    return MOK_OK;
}

// ------------------------------------------------------------------ expert parallelism
// Scratch of one rank's expert phase: its sorted rows, the token rows it
// pulled and the h of those rows, sized for the largest share it can receive
// (every token of every rank choosing min(k, E_loc) of its experts).
struct EpScratch {
    int *seg, *offsets, *gorder, *row_token, *row_slot, *row_gdst;
    int *recv_idx, *uniq_src, *n_recv;   // the distinct (source rank, token) rows received
    float *row_w;
    float **push;                   // [kEpMaxRanks] every rank's fp32 slot rows (forward push)
    float **push_dx;                // [kEpMaxRanks] every rank's fp32 dX slot rows (backward push)
    float **push_g;                 // [kEpMaxRanks] every rank's slot-gradient partials
    int *sched;                     // [kSchedCounters] tile counters
    int *ready;                     // [n_mtiles] per-M-tile readiness (persistent experts phase)
    int *zero;                      // sched and ready: the counters the persistent phase zeroes
    int n_zero;
    unsigned long long *gs_flags;   // grid-barrier tags, release tag, epoch
    int *mt_base;                   // [G + 1] first 128-row M tile of each group (persistent backward phase)
    __nv_bfloat16 *x_recv, *h;
    __nv_bfloat16 *gu, *hw;         // training: saved g/u and w h of the owner's rows
    __nv_bfloat16 *dy_recv, *dgu;   // training: pulled dy rows, dGU
    float *gpart;                   // training: slot-gradient partials of the owner's routed rows
    uint8_t *xq_recv, *xs_recv;     // MXFP8: pulled e4m3 x rows and their scales
    uint8_t *hq, *hs;               // MXFP8: h codes and scales
    uint8_t *dyq_recv, *dys_recv;   // MXFP8 training: the pulled dy rows quantised
    uint8_t *dguq, *dgus;           // MXFP8 training: dGU codes and scales
    long long rr_cap, rows_cap;
    long long n_pull;               // received token rows at most: world T
    size_t bytes;
};

EpScratch carve_ep(const moe_cfg &c, int world, bool training, void *buf)
{
    const Shapes s = shapes(c);
    const long long el = s.E / world;
    EpScratch e{};
    e.rr_cap = static_cast<long long>(world) * s.T * std::min<long long>(s.k, el);
    e.rows_cap = e.rr_cap + s.S * s.T;
    e.n_pull = static_cast<long long>(world) * s.T;
    Carver cv(buf);
    e.seg = cv.take<int>(s.E + 1);
    e.offsets = cv.take<int>(el + s.S + 1);
    e.gorder = cv.take<int>(el + s.S);
    e.row_token = cv.take<int>(e.rows_cap);
    e.recv_idx = cv.take<int>(static_cast<long long>(world) * s.T);
    e.uniq_src = cv.take<int>(static_cast<long long>(world) * s.T);
    e.n_recv = cv.take<int>(1);
    e.row_slot = cv.take<int>(e.rows_cap);
    e.row_gdst = cv.take<int>(e.rr_cap);
    e.row_w = cv.take<float>(e.rows_cap);
    e.push = cv.take<float *>(kEpMaxRanks);
    e.push_dx = cv.take<float *>(kEpMaxRanks);
    e.push_g = cv.take<float *>(kEpMaxRanks);
    const int n_mtiles = static_cast<int>(e.rows_cap / BM + el + s.S + 1);
    e.n_zero = kSchedCounters + n_mtiles;
    e.zero = cv.take<int>(e.n_zero);
    e.sched = e.zero;
    e.ready = e.zero + kSchedCounters;
    e.gs_flags = cv.take<unsigned long long>(kMaxFusedCtas + 2);
    e.mt_base = cv.take<int>(el + s.S + 1);
    if (c.dtype == MOK_DTYPE_MXFP8) {
        e.xq_recv = cv.take<uint8_t>((s.T + e.n_pull) * s.H);
        e.xs_recv = cv.take<uint8_t>((s.T + e.n_pull) * s.H / 32);
        e.hq = cv.take<uint8_t>(e.rows_cap * s.I);
        e.hs = cv.take<uint8_t>(e.rows_cap * s.I / 32);
        if (training) {
            // forward: g/u, the dequantised h, w Q(h); backward: the decoded x rows, the
            // pulled dy rows and their quantisation, dGU in bf16 and MXFP8, the partials
            e.gu = cv.take<__nv_bfloat16>(e.rows_cap * 2 * s.I);
            e.h = cv.take<__nv_bfloat16>(e.rows_cap * s.I);
            e.hw = cv.take<__nv_bfloat16>(e.rows_cap * s.I);
            e.x_recv = cv.take<__nv_bfloat16>((s.T + e.n_pull) * s.H);
            e.dy_recv = cv.take<__nv_bfloat16>((s.T + e.n_pull) * s.H);
            e.dyq_recv = cv.take<uint8_t>((s.T + e.n_pull) * s.H);
            e.dys_recv = cv.take<uint8_t>((s.T + e.n_pull) * s.H / 32);
            e.dgu = cv.take<__nv_bfloat16>(e.rows_cap * 2 * s.I);
            e.dguq = cv.take<uint8_t>(e.rows_cap * 2 * s.I);
            e.dgus = cv.take<uint8_t>(e.rows_cap * 2 * s.I / 32);
            e.gpart = cv.take<float>(e.rr_cap * (s.I / 128));
        }
        e.bytes = align_up(cv.off, 256);
        return e;
    }
    e.x_recv = cv.take<__nv_bfloat16>((s.T + e.n_pull) * s.H);
    e.h = cv.take<__nv_bfloat16>(e.rows_cap * s.I);
    if (training) {
        e.gu = cv.take<__nv_bfloat16>(e.rows_cap * 2 * s.I);
        e.hw = cv.take<__nv_bfloat16>(e.rows_cap * s.I);
        e.dy_recv = cv.take<__nv_bfloat16>((s.T + e.n_pull) * s.H);
        e.dgu = cv.take<__nv_bfloat16>(e.rows_cap * 2 * s.I);
        e.gpart = cv.take<float>(e.rr_cap * (s.I / 128));
    }
    e.bytes = align_up(cv.off, 256);
    return e;
}

// A rank's buffer of the backward's token side: what the owners push to it (the
// dX slot rows and the slot-gradient partials of its routed rows) and what it
// computes from them.
struct EpSrcBwd {
    float *dl, *gpart, *partial, *dxs;
    size_t bytes;
};

EpSrcBwd carve_ep_src_bwd(const moe_cfg &c, void *buf)
{
    const Shapes s = shapes(c);
    Carver cv(buf);
    EpSrcBwd b{};
    b.dl = cv.take<float>(s.TK);
    b.gpart = cv.take<float>(s.TK * (s.I / 128));
    b.partial = cv.take<float>(s.max_chunks * s.H);
    b.dxs = cv.take<float>(s.T * s.kk * s.H);
    b.bytes = align_up(cv.off, 256);
    return b;
}

int check_ep(const moe_cfg *c, int world, int rank)
{
    MOK_TRY(check_cfg(c));
    if (world < 1 || world > kEpMaxRanks || rank < 0 || rank >= world || c->E % world) return MOK_ERR_INVALID;
    if (static_cast<long long>(c->T) * (c->top_k + c->n_shared) >= (1ll << kEpRankShift)) return MOK_ERR_INVALID;
    const long long rows = static_cast<long long>(world) * c->T * std::min(c->top_k, c->E / world) +
                           static_cast<long long>(c->n_shared + 1) * c->T;
    if (rows >= (1ll << 31)) return MOK_ERR_INVALID;
    return MOK_OK;
}

int ep_route(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const DeviceInfo &dev,
             cudaStream_t stream)
{
    t_launches = 0;
    t_pdl = false;
    FwdPlan pl;
    MOK_TRY(build_route_plan(c, x, p, st, dev, pl));
    if (const cudaError_t e = cudaMemsetAsync(st.sched, 0, kSchedCounters * sizeof(int), stream); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaMemsetAsync(tile counters)", e);
    MOK_TRY(launch_router(c, p, st, dev, pl, stream));
    MOK_TRY(launch_dispatch(pl, stream));
    if (c.dtype != MOK_DTYPE_MXFP8) return MOK_OK;
    // MXFP8: the rank's x codes and scales, which the owners pull
    const long long xb = static_cast<long long>(c.T) * c.H / 32;
    return launch_k(quantize_mxfp8_kernel, dim3(blocks_for(xb, 256)), dim3(256), 0, stream, "quantize_mxfp8_kernel",
                    static_cast<const __nv_bfloat16 *>(x), xb, st.xq, st.xs, static_cast<long long>(c.H / 32), 0ll,
                    static_cast<__nv_bfloat16 *>(nullptr));
}

// Tensor maps and arguments of an owner's two expert GEMMs.
struct EpGemms {
    CUtensorMap gB, gBs, gO, gO2, gO3, dA, dB, dBs, dO;
    GemmArgs ga, gd;
};

// MXFP8 (inference): gate/up on the pulled x codes with the SwiGLU epilogue
// requantising h, down with the push epilogue storing bf16 rows into the slot
// rows of the tokens' ranks.
int ep_plan_mx(const moe_cfg &c, int el, bool training, const moe_params &p, const State &own, const EpScratch &es,
               const DeviceInfo &dev, EpGemms &q)
{
    const Shapes s = shapes(c);
    if (!make_tmap(&q.gB, p.w_gate_up, s.H, el * 2 * s.I, 128, 128, 1) ||
        !make_tmap(&q.gBs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : el) * 2 * s.I, 128, 128, 1) ||
        !make_tmap(&q.gO, es.hq, s.I, es.rows_cap, 128, 32, 1) ||
        !make_tmap(&q.dA, es.hq, s.I, es.rows_cap, 128, 128, 1) ||
        !make_tmap(&q.dB, p.w_down, s.I, el * s.H, 128, 256, 1) ||
        !make_tmap(&q.dBs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : el) * s.H, 128, 256, 1) ||
        !make_tmap(&q.dO, own.O, s.H, s.T * s.kk, 64, 1, 2))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel MXFP8 GEMMs)");
    q.gO2 = q.gO3 = q.gO;
    GemmArgs &ga = q.ga;
    ga = GemmArgs{};
    ga.sched = es.sched + 0;
    ga.num_groups = el + c.n_shared;
    ga.num_routed = el;
    ga.offsets = es.offsets;
    ga.row_token = es.row_token;
    ga.row_slot = es.row_slot;
    ga.row_w = es.row_w;
    ga.n_tiles = c.I / 128;
    ga.num_kb = c.H / 128;
    ga.b_rows_per_group = 2 * c.I;
    ga.b_half = c.I;
    ga.inter = c.I;
    ga.gather_src = reinterpret_cast<const __nv_bfloat16 *>(es.xq_recv);
    ga.gather_ld = c.H;
    ga.out = reinterpret_cast<__nv_bfloat16 *>(es.hq);
    ga.out_scales = es.hs;
    ga.out2 = training ? es.gu : nullptr;       // training: g/u, the dequantised h, w Q(h)
    ga.out_hb = training ? es.h : nullptr;
    ga.out3 = training ? es.hw : nullptr;
    ga.sfa_src = es.xs_recv;
    ga.sfb_src = p.s_gate_up;
    ga.sfb_src_s = s.S ? p.ss_gate_up : p.s_gate_up;
    ga.sf_ld = c.H / 32;
    ga.sfb_row_tiles = static_cast<int>(el * 2 * s.I / 128);
    ga.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : el) * 2 * s.I / 128);
    ga.status = dev.status;
    GemmArgs &gd = q.gd;
    gd = ga;
    gd.sched = es.sched + 1;
    gd.n_tiles = c.H / 256;
    gd.num_kb = c.I / 128;
    gd.b_rows_per_group = c.H;
    gd.b_half = 0;
    gd.out = reinterpret_cast<__nv_bfloat16 *>(own.O);
    gd.out_scales = nullptr;
    gd.out2 = gd.out3 = gd.out_hb = nullptr;
    gd.ldo = c.H;
    gd.gather_src = nullptr;
    gd.push_dst = es.push;
    gd.sfa_src = es.hs;
    gd.sfb_src = p.s_down;
    gd.sfb_src_s = s.S ? p.ss_down : p.s_down;
    gd.sf_ld = c.I / 32;
    gd.sfb_row_tiles = static_cast<int>(el * s.H / 128);
    gd.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : el) * s.H / 128);
    return MOK_OK;
}

// BF16: gate/up on the pulled x rows with the SwiGLU epilogue (training: also g/u
// and w h), down with the push epilogue storing fp32 rows into the slot rows of
// the tokens' ranks (the map over the owner's own slot rows only has to exist).
int ep_plan_bf16(const moe_cfg &c, int el, bool training, const moe_params &p, const State &own,
                 const EpScratch &es, const DeviceInfo &dev, EpGemms &q)
{
    const Shapes s = shapes(c);
    if (!make_tmap(&q.gB, p.w_gate_up, s.H, el * 2 * s.I, BK, 128, 2) ||
        !make_tmap(&q.gBs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : el) * 2 * s.I, BK, 128, 2) ||
        !make_tmap(&q.gO, es.h, s.I, es.rows_cap, 64, 32, 2) ||
        !make_tmap(&q.gO2, training ? es.gu : es.h, training ? 2 * s.I : s.I, es.rows_cap, 64, 32, 2) ||
        !make_tmap(&q.gO3, training ? es.hw : es.h, s.I, es.rows_cap, 64, 32, 2) ||
        !make_tmap(&q.dA, es.h, s.I, es.rows_cap, BK, 128, 2) ||
        !make_tmap(&q.dB, p.w_down, s.I, el * s.H, BK, 256, 2) ||
        !make_tmap(&q.dBs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : el) * s.H, BK, 256, 2) ||
        !make_tmap(&q.dO, own.O, s.H, s.T * s.kk, 32, 1, 4))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel GEMMs)");
    GemmArgs &ga = q.ga;
    ga = GemmArgs{};
    ga.sched = es.sched + 0;
    ga.num_groups = el + c.n_shared;
    ga.num_routed = el;
    ga.offsets = es.offsets;
    ga.row_token = es.row_token;
    ga.row_slot = es.row_slot;
    ga.row_w = es.row_w;
    ga.n_tiles = c.I / 128;
    ga.num_kb = c.H / BK;
    ga.b_rows_per_group = 2 * c.I;
    ga.b_half = c.I;
    ga.inter = c.I;
    ga.gather_src = es.x_recv;
    ga.gather_ld = c.H;
    ga.out = es.h;
    ga.out2 = training ? es.gu : nullptr;
    ga.out3 = training ? es.hw : nullptr;
    ga.status = dev.status;
    GemmArgs &gd = q.gd;
    gd = ga;
    gd.sched = es.sched + 1;
    gd.n_tiles = c.H / 256;
    gd.num_kb = c.I / BK;
    gd.b_rows_per_group = c.H;
    gd.b_half = 0;
    gd.out = nullptr;
    gd.out2 = gd.out3 = nullptr;
    gd.out_f32 = own.O;
    gd.push_dst = es.push;
    gd.ldo = c.H;
    return MOK_OK;
}

// Fill one pull of rows of `row_bytes` bytes from every rank's src matrix (src[s]:
// rank s's [T, row_bytes] rows) into dst: the owner's own T rows, then each
// received row.
int make_pull(EpPull &a, int &unit16, const void *const *src, int world, int rank, void *dst, long long row_bytes,
              const EpScratch &es, const moe_cfg &c, const DeviceInfo &dev);

int launch_pull(const void *const *src, int world, int rank, void *dst, long long row_bytes, const EpScratch &es,
                const moe_cfg &c, const DeviceInfo &dev, cudaStream_t stream)
{
    EpPull a;
    int unit16 = 0;
    MOK_TRY(make_pull(a, unit16, src, world, rank, dst, row_bytes, es, c, dev));
    return unit16 ? launch_k(ep_pull_kernel<uint4>, dim3(dev.sms * 8), dim3(256), 0, stream, "ep_pull_kernel", a)
                  : launch_k(ep_pull_kernel<uint2>, dim3(dev.sms * 8), dim3(256), 0, stream, "ep_pull_kernel", a);
}

int make_pull(EpPull &a, int &unit16, const void *const *src, int world, int rank, void *dst, long long row_bytes,
              const EpScratch &es, const moe_cfg &c, const DeviceInfo &dev)
{
    a = EpPull{};
    for (int r = 0; r < world; ++r) a.src[r] = static_cast<const uint8_t *>(src[r]);
    a.dst = static_cast<uint8_t *>(dst);
    a.row_bytes = row_bytes;
    a.T = c.T; a.world = world; a.rank = rank;
    a.n_recv = es.n_recv;
    a.row_src = es.uniq_src;
    a.status = dev.status;
    if (row_bytes % 8) return fail(MOK_ERR_INVALID, "expert-parallel pull: rows of a multiple of 8 bytes");
    unit16 = row_bytes % 16 == 0;
    return MOK_OK;
}

// The persistent experts phase: one cooperative launch (ep_fused.cuh).  src0/src1:
// the ranks' x rows (BF16), or their x codes and x scales (MXFP8).
template <bool MX>
int launch_ep_fused(const moe_cfg &c, int world, int rank, const void *const *src0, const void *const *src1,
                    const EpView &v, const EpArgs &ea, const EpScratch &es, const EpGemms &q, const DeviceInfo &dev,
                    cudaStream_t stream)
{
    using F = FusedCfg<MX>;
    if (dev.sms > kMaxFusedCtas) return fail(MOK_ERR_UNSUPPORTED, "more SMs than the grid barrier holds");
    EpFusedArgs a{};
    a.gs.flags = es.gs_flags;
    a.gs.go = es.gs_flags + kMaxFusedCtas;
    a.gs.epoch = es.gs_flags + kMaxFusedCtas + 1;
    a.status = dev.status;
    a.zero = es.zero;
    a.n_zero = es.n_zero;
    a.v = v;
    a.ea = ea;
    if (MX) {
        a.n_pull = 2;
        MOK_TRY(make_pull(a.pull[0], a.pull16[0], src0, world, rank, es.xq_recv, c.H, es, c, dev));
        MOK_TRY(make_pull(a.pull[1], a.pull16[1], src1, world, rank, es.xs_recv, c.H / 32, es, c, dev));
    } else {
        a.n_pull = 1;
        MOK_TRY(make_pull(a.pull[0], a.pull16[0], src0, world, rank, es.x_recv, 2ll * c.H, es, c, dev));
    }
    a.ga = q.ga;
    a.gd = q.gd;
    a.ga.ready = a.gd.ready = es.ready;
    a.ga.ready_role = kReadySignal;
    a.gd.ready_role = kReadyWait;
    a.gd.ready_target = 4 * (c.I / 128);    // four epilogue warps per gate/up tile, I/128 tiles per M tile
    FusedMaps m{};
    m.gB = q.gB; m.gBs = q.gBs; m.gO = q.gO; m.gO2 = q.gO2; m.gO3 = q.gO3;
    m.dA = q.dA; m.dB = q.dB; m.dBs = q.dBs; m.dO = q.dO;
    m.rA = m.rB = m.rO = q.gB;                // unused by this kernel
    cudaError_t e = cudaFuncSetAttribute(moe_ep_experts_fused_kernel<MX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         F::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(moe_ep_experts_fused_kernel)", e);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(dev.sms));
    lc.blockDim = dim3(kFusedThreads);
    lc.dynamicSmemBytes = F::SMEM_BYTES;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, moe_ep_experts_fused_kernel<MX>, m, a);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaLaunchKernelEx(moe_ep_experts_fused_kernel, cooperative)", e);
    ++t_launches;
    return MOK_OK;
}

int ep_experts(const moe_cfg &c, int world, int rank, bool training, const void *const *xr, void *const *sr,
               const moe_params &p, const EpScratch &es, const DeviceInfo &dev, cudaStream_t stream)
{
    t_launches = 0;
    t_pdl = false;
    const Shapes s = shapes(c);
    const int el = c.E / world;
    EpView v{};
    for (int r = 0; r < world; ++r) {
        const State q = carve_state(c, sr[r], false);
        v.counts[r] = q.counts;
        v.offsets[r] = q.offsets;
        v.perm[r] = q.perm;
        v.topk_w[r] = q.topk_w;
        v.topk_idx[r] = q.topk_idx;
        v.O[r] = q.O;
    }
    EpArgs a{};
    a.world = world; a.rank = rank;
    a.T = c.T; a.H = c.H; a.k = c.top_k; a.kk = static_cast<int>(s.kk); a.S = c.n_shared; a.E_loc = el;
    a.rr_cap = static_cast<int>(es.rr_cap);
    a.seg = es.seg; a.offsets = es.offsets;
    a.row_token = es.row_token; a.row_slot = es.row_slot; a.row_w = es.row_w;
    a.recv_idx = es.recv_idx; a.uniq_src = es.uniq_src; a.n_recv = es.n_recv;
    a.row_gdst = es.row_gdst; a.gorder = es.gorder;
    a.push = es.push; a.status = dev.status;

    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    const State own = carve_state(c, sr[rank], false);
    EpGemms q;
    MOK_TRY(mx ? ep_plan_mx(c, el, training, p, own, es, dev, q) : ep_plan_bf16(c, el, training, p, own, es, dev, q));
    if (t_schedule == MOK_SCHEDULE_PERSISTENT) {
        const void *xq[kEpMaxRanks] = {}, *xs[kEpMaxRanks] = {};
        if (mx)
            for (int r = 0; r < world; ++r) {
                const State st_r = carve_state(c, sr[r], false);
                xq[r] = st_r.xq;
                xs[r] = st_r.xs;
            }
        return mx ? launch_ep_fused<true>(c, world, rank, xq, xs, v, a, es, q, dev, stream)
                  : launch_ep_fused<false>(c, world, rank, xr, nullptr, v, a, es, q, dev, stream);
    }

    if (const cudaError_t e = cudaMemsetAsync(es.sched, 0, kSchedCounters * sizeof(int), stream); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaMemsetAsync(tile counters)", e);
    MOK_TRY(launch_k(ep_layout_kernel, dim3(1), dim3(256), 0, stream, "ep_layout_kernel", v, a));
    MOK_TRY(launch_k(ep_unique_kernel, dim3(1), dim3(1024), 0, stream, "ep_unique_kernel", v, a));
    MOK_TRY(launch_k(ep_rows_kernel, dim3(static_cast<unsigned>(c.E + c.n_shared * blocks_for(c.T, 256))), dim3(256), 0,
                     stream, "ep_rows_kernel", v, a));
    if (mx) {
        // pull the x codes and scales each rank quantised in its routing phase
        const void *xq[kEpMaxRanks], *xs[kEpMaxRanks];
        for (int r = 0; r < world; ++r) {
            const State st_r = carve_state(c, sr[r], false);
            xq[r] = st_r.xq;
            xs[r] = st_r.xs;
        }
        MOK_TRY(launch_pull(xq, world, rank, es.xq_recv, c.H, es, c, dev, stream));
        MOK_TRY(launch_pull(xs, world, rank, es.xs_recv, c.H / 32, es, c, dev, stream));
        MOK_TRY(launch_gemm<typename FusedCfg<true>::GateUp>(q.gB, q.gB, q.gBs, q.gO, q.gO2, q.gO3, q.ga, dev.sms,
                                                            stream));
        return launch_gemm<typename FusedCfg<true>::Down>(q.dA, q.dB, q.dBs, q.dO, q.dO, q.dO, q.gd, dev.sms, stream);
    }
    MOK_TRY(launch_pull(xr, world, rank, es.x_recv, 2ll * c.H, es, c, dev, stream));
    MOK_TRY(launch_gemm<typename FusedCfg<false>::GateUp>(q.gB, q.gB, q.gBs, q.gO, q.gO2, q.gO3, q.ga, dev.sms, stream));
    return launch_gemm<typename FusedCfg<false>::Down>(q.dA, q.dB, q.dBs, q.dO, q.dO, q.dO, q.gd, dev.sms, stream);
}

// The persistent backward experts phase: one cooperative launch (ep_fused.cuh).
template <bool N256, bool MX>
int launch_ep_bwd_fused(const moe_cfg &c, int world, int rank, const void *const *dyr, const EpTable &tdx,
                        const EpTable &tg, const EpScratch &es, const FusedBwdMaps &m, const GemmArgs &g1,
                        const GemmArgs &g2, const GemmArgs &g3, const GemmArgs &g4, int g2_units, int g4_units,
                        const EpMxPrep &prep, const DeviceInfo &dev, cudaStream_t stream)
{
    using F = FusedBwdCfg<N256, MX>;
    if (dev.sms > kMaxFusedCtas) return fail(MOK_ERR_UNSUPPORTED, "more SMs than the grid barrier holds");
    EpBwdFusedArgs a{};
    a.gs.flags = es.gs_flags;
    a.gs.go = es.gs_flags + kMaxFusedCtas;
    a.gs.epoch = es.gs_flags + kMaxFusedCtas + 1;
    a.status = dev.status;
    a.zero = es.zero;
    a.n_zero = es.n_zero;
    MOK_TRY(make_pull(a.pull, a.pull16, dyr, world, rank, es.dy_recv, 2ll * c.H, es, c, dev));
    a.tdx = tdx;
    a.tg = tg;
    a.push_dx = es.push_dx;
    a.push_g = es.push_g;
    a.world = world;
    a.g1 = g1;
    a.g1.ready = es.ready;
    a.g1.ready_role = kReadySignal;
    a.g2 = a.g2r = g2;
    a.g3 = g3;
    a.g3.ready = es.ready;
    a.g3.ready_role = kReadyWait;
    a.g3.ready_target = 4 * g1.n_tiles;     // four epilogue warps per down-dgrad tile, its N tiles per M tile
    a.g4 = a.g4r = g4;
    a.g4.ready = a.g4r.ready = es.ready;
    a.g4.ready_role = a.g4r.ready_role = kReadyWaitGroup;
    a.g4.ready_target = a.g4r.ready_target = 4 * g1.n_tiles;
    a.g4.mt_base = a.g4r.mt_base = es.mt_base;
    a.g2_units = g2_units;
    a.g4_units = g4_units;
    a.offsets_all = es.offsets;
    a.mt_base = es.mt_base;
    a.gpart = es.gpart;
    a.row_gdst = es.row_gdst;
    a.seg = es.seg;
    a.n_seg = c.E;
    a.nt = g1.n_tiles;
    a.tk = c.T * c.top_k;
    a.prep = prep;
    cudaError_t e = cudaFuncSetAttribute(moe_ep_bwd_experts_fused_kernel<N256, MX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM_BYTES);
    if (e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaFuncSetAttribute(moe_ep_bwd_experts_fused_kernel)", e);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(dev.sms));
    lc.blockDim = dim3(kFusedThreads);
    lc.dynamicSmemBytes = F::SMEM_BYTES;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, moe_ep_bwd_experts_fused_kernel<N256, MX>, m, a);
    if (e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaLaunchKernelEx(moe_ep_bwd_experts_fused_kernel, cooperative)", e);
    ++t_launches;
    return MOK_OK;
}

// Backward, owner side: pull dy rows, down dgrad (SwiGLU backward, slot-gradient
// partials pushed to the rows' ranks), gate/up dgrad (dX rows pushed into the
// dX slot rows of the tokens' ranks), both weight gradients of the owner's experts
// (and this rank's share of the shared experts'), from the rows the forward kept.
int ep_bwd_experts(const moe_cfg &c, int world, int rank, const void *const *dyr, void *const *br,
                   const moe_params &p, const moe_grads &gr, const EpScratch &es, const DeviceInfo &dev,
                   cudaStream_t stream)
{
    t_launches = 0;
    t_pdl = false;
    const Shapes s = shapes(c);
    const int el = c.E / world;
    const long long G = el + s.S;
    const bool n256 = c.I % 256 == 0;
    const bool mx = c.dtype == MOK_DTYPE_MXFP8;
    EpTable tdx{}, tg{};
    for (int r = 0; r < world; ++r) {
        const EpSrcBwd q = carve_ep_src_bwd(c, br[r]);
        tdx.p[r] = q.dxs;
        tg.p[r] = q.gpart;
    }
    const EpSrcBwd own = carve_ep_src_bwd(c, br[rank]);

    GemmArgs base{};
    base.num_groups = static_cast<int>(G);
    base.num_routed = el;
    base.offsets = es.offsets;
    base.gorder = es.gorder;
    base.row_token = es.row_token;
    base.row_slot = es.row_slot;
    base.row_w = es.row_w;
    base.inter = c.I;
    base.gather_src = es.dy_recv;
    base.gather_ld = c.H;
    base.status = dev.status;

    FusedBwdMaps m;
    // down dgrad: dh = w (dy W_down), SwiGLU backward -> dGU, slot-gradient partials
    // (MXFP8: on the quantised dy rows against W_down^T quantised along H)
    if (!(mx ? make_tmap(&m.d1B, p.wt_down, s.H, el * s.I, 128, 256, 1) &&
                   make_tmap(&m.d1Bs, s.S ? p.wst_down : p.wt_down, s.H, (s.S ? s.S : el) * s.I, 128, 256, 1)
             : make_tmap(&m.d1B, p.w_down, s.I, el * s.H, 64, 64, 2) &&
                   make_tmap(&m.d1Bs, s.S ? p.ws_down : p.w_down, s.I, (s.S ? s.S : el) * s.H, 64, 64, 2)) ||
        !make_tmap(&m.d1O, es.dgu, 2 * s.I, es.rows_cap, 64, 32, 2))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel down dgrad)");
    GemmArgs g1 = base;
    g1.sched = es.sched + 2;
    g1.num_kb = c.H / BK;
    g1.b_rows_per_group = c.H;
    g1.aux = es.gu;
    g1.aux_h = es.h;
    g1.gpart = es.gpart;
    g1.out = es.dgu;
    g1.n_tiles = n256 ? c.I / 256 : c.I / 128;
    if (mx) {
        g1.num_kb = c.H / 128;
        g1.b_rows_per_group = c.I;
        g1.gather_src = reinterpret_cast<const __nv_bfloat16 *>(es.dyq_recv);
        g1.sfa_src = es.dys_recv;
        g1.sf_ld = c.H / 32;
        g1.sfb_src = p.st_down;
        g1.sfb_src_s = s.S ? p.sst_down : p.st_down;
        g1.sfb_row_tiles = static_cast<int>(el * s.I / 128);
        g1.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : el) * s.I / 128);
        g1.out_q = es.dguq;
        g1.out_scales = es.dgus;
    }

    // down wgrad: dW_down[g] = sum_r dy[token r]^T (w_r h_r)
    if (!make_tmap(&m.w2O, gr.dw_down, s.I, el * s.H, 64, 32, 2) ||
        !make_tmap(&m.w2O2, s.S ? gr.dws_down : gr.dw_down, s.I, (s.S ? s.S : el) * s.H, 64, 32, 2) ||
        !make_tmap(&m.w2B, es.hw, s.I, es.rows_cap, 64, 64, 2))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel down wgrad)");
    GemmArgs g2 = base;
    g2.sched = es.sched + 3;
    g2.m_tiles = c.H / 128;
    g2.out = static_cast<__nv_bfloat16 *>(gr.dw_down);
    g2.out_s = static_cast<__nv_bfloat16 *>(gr.dws_down);
    g2.ldo = c.I;
    g2.group_out_elems = s.H * s.I;
    int g2_units = 0;
    if (n256) {
        g2.n_tiles = c.I / 256;
        g2.k_split = kResidentRows;
        g2.m_per_unit = resident_m_per_unit(g2.m_tiles);
        g2_units = static_cast<int>(G * g2.n_tiles * ((g2.m_tiles + g2.m_per_unit - 1) / g2.m_per_unit));
    } else {
        g2.n_tiles = c.I / 128;
    }
    const long long t2 = G * g2.m_tiles * g2.n_tiles;
    const int g2_grid = static_cast<int>(t2 < dev.sms ? t2 : dev.sms);

    // gate/up dgrad: dX rows = dGU W_gate_up, pushed into the tokens' ranks
    if (!(mx ? make_tmap(&m.d3A, es.dguq, 2 * s.I, es.rows_cap, 128, 128, 1) &&
                   make_tmap(&m.d3B, p.wt_gate_up, 2 * s.I, el * s.H, 128, 256, 1) &&
                   make_tmap(&m.d3Bs, s.S ? p.wst_gate_up : p.wt_gate_up, 2 * s.I, (s.S ? s.S : el) * s.H, 128, 256, 1)
             : make_tmap(&m.d3A, es.dgu, 2 * s.I, es.rows_cap, BK, 128, 2) &&
                   make_tmap(&m.d3B, p.w_gate_up, s.H, el * 2 * s.I, 64, 64, 2) &&
                   make_tmap(&m.d3Bs, s.S ? p.ws_gate_up : p.w_gate_up, s.H, (s.S ? s.S : el) * 2 * s.I, 64, 64, 2)) ||
        !make_tmap(&m.d3O, own.dxs, s.H, s.T * s.kk, 32, 1, 4))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel gate/up dgrad)");
    GemmArgs g3 = base;
    g3.sched = es.sched + 4;
    g3.n_tiles = c.H / 256;
    g3.num_kb = 2 * c.I / BK;
    g3.b_rows_per_group = 2 * c.I;
    g3.out_f32 = own.dxs;
    g3.push_dst = es.push_dx;
    g3.ldo = c.H;
    if (mx) {
        g3.num_kb = 2 * c.I / 128;
        g3.b_rows_per_group = c.H;
        g3.gather_src = nullptr;
        g3.sfa_src = es.dgus;
        g3.sf_ld = 2 * c.I / 32;
        g3.sfb_src = p.st_gate_up;
        g3.sfb_src_s = s.S ? p.sst_gate_up : p.st_gate_up;
        g3.sfb_row_tiles = static_cast<int>(el * s.H / 128);
        g3.sfb_row_tiles_s = static_cast<int>((s.S ? s.S : el) * s.H / 128);
    }

    // gate/up wgrad: dW_gate_up[g] = sum_r dGU_r^T x[token r] (the pulled x rows)
    if (!make_tmap(&m.w4A, es.dgu, 2 * s.I, es.rows_cap, 64, 64, 2) ||
        !make_tmap(&m.w4O, gr.dw_gate_up, s.H, el * 2 * s.I, 64, 32, 2) ||
        !make_tmap(&m.w4O2, s.S ? gr.dws_gate_up : gr.dw_gate_up, s.H, (s.S ? s.S : el) * 2 * s.I, 64, 32, 2))
        return fail(MOK_ERR_INVALID, "tensor map (expert-parallel gate/up wgrad)");
    GemmArgs g4 = base;
    g4.sched = es.sched + 5;
    g4.gather_src = es.x_recv;
    g4.m_tiles = 2 * c.I / 128;
    g4.n_tiles = c.H / 256;
    g4.out = static_cast<__nv_bfloat16 *>(gr.dw_gate_up);
    g4.out_s = static_cast<__nv_bfloat16 *>(gr.dws_gate_up);
    g4.ldo = c.H;
    g4.group_out_elems = 2 * s.I * s.H;
    g4.k_split = kResidentRows;
    g4.m_per_unit = resident_m_per_unit(g4.m_tiles);
    const long long t4 = G * g4.m_tiles * g4.n_tiles;
    const int g4_grid = static_cast<int>(t4 < dev.sms ? t4 : dev.sms);
    const int g4_units = static_cast<int>(G * g4.n_tiles * ((g4.m_tiles + g4.m_per_unit - 1) / g4.m_per_unit));

    EpMxPrep prep{};                         // MXFP8: quantise the pulled dy rows, decode the x codes
    prep.dy = es.dy_recv;
    prep.dyq = es.dyq_recv;
    prep.dys = es.dys_recv;
    prep.xq = es.xq_recv;
    prep.xs = es.xs_recv;
    prep.xdq = es.x_recv;
    prep.n_recv = es.n_recv;
    prep.T = c.T; prep.world = world; prep.H = c.H;
    if (t_schedule == MOK_SCHEDULE_PERSISTENT) {
        if (mx)
            return launch_ep_bwd_fused<true, true>(c, world, rank, dyr, tdx, tg, es, m, g1, g2, g3, g4, g2_units,
                                                   g4_units, prep, dev, stream);
        return n256 ? launch_ep_bwd_fused<true, false>(c, world, rank, dyr, tdx, tg, es, m, g1, g2, g3, g4, g2_units,
                                                       g4_units, prep, dev, stream)
                    : launch_ep_bwd_fused<false, false>(c, world, rank, dyr, tdx, tg, es, m, g1, g2, g3, g4, g2_units,
                                                        g4_units, prep, dev, stream);
    }
    if (const cudaError_t e = cudaMemsetAsync(es.sched, 0, kSchedCounters * sizeof(int), stream); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaMemsetAsync(tile counters)", e);
    MOK_TRY(launch_k(ep_table_kernel, dim3(1), dim3(32), 0, stream, "ep_table_kernel", tdx, es.push_dx, world));
    MOK_TRY(launch_k(ep_table_kernel, dim3(1), dim3(32), 0, stream, "ep_table_kernel", tg, es.push_g, world));
    MOK_TRY(launch_pull(dyr, world, rank, es.dy_recv, 2ll * c.H, es, c, dev, stream));
    if (mx) {
        MOK_TRY(launch_k(ep_mx_prepare_kernel, dim3(dev.sms * 8), dim3(256), 0, stream, "ep_mx_prepare_kernel", prep));
        MOK_TRY(launch_gemm<DgradDownMX>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1, dev.sms, stream));
    } else if (n256)
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::DgradDown>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1,
                                                                  dev.sms, stream));
    else
        MOK_TRY(launch_gemm<typename FusedBwdCfg<false>::DgradDown>(m.d1B, m.d1B, m.d1Bs, m.d1O, m.d1O, m.d1O, g1,
                                                                   dev.sms, stream));
    MOK_TRY(launch_k(ep_push_gpart_kernel, dim3(dev.sms), dim3(256), 0, stream, "ep_push_gpart_kernel",
                     static_cast<const float *>(es.gpart), static_cast<const int *>(es.row_gdst),
                     static_cast<const int *>(es.seg), c.E, g1.n_tiles, es.push_g, world, c.T * c.top_k, dev.status));
    if (n256) {
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::WgradDown>(m.w2B, m.w2B, m.w2B, m.w2O, m.w2O2, m.w2O, g2,
                                                                  g2_grid, stream));
        MOK_TRY(launch_wgrad_resident<WgradResCfg<true>>(m.w2B, m.w2B, m.w2O, m.w2O2, g2,
                                                         g2_units < dev.sms ? g2_units : dev.sms, stream));
    } else {
        MOK_TRY(launch_gemm<typename FusedBwdCfg<false>::WgradDown>(m.w2B, m.w2B, m.w2B, m.w2O, m.w2O2, m.w2O, g2,
                                                                   g2_grid, stream));
    }
    if (mx)
        MOK_TRY(launch_gemm<DgradGUMX>(m.d3A, m.d3B, m.d3Bs, m.d3O, m.d3O, m.d3O, g3, dev.sms, stream));
    else
        MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::DgradGU>(m.d3A, m.d3B, m.d3Bs, m.d3O, m.d3O, m.d3O, g3,
                                                                dev.sms, stream));
    MOK_TRY(launch_gemm<typename FusedBwdCfg<true>::WgradGU>(m.w4A, m.w4A, m.w4A, m.w4O, m.w4O2, m.w4O, g4, g4_grid,
                                                            stream));
    return launch_wgrad_resident<WgradResCfg<false>>(m.w4A, m.w4A, m.w4O, m.w4O2, g4,
                                                     g4_units < dev.sms ? g4_units : dev.sms, stream);
}

// Backward, token side: slot gradients from the partials the owners pushed, the
// router gradient of this rank's tokens, dx from the dX slot rows they pushed.
int ep_bwd_combine(const moe_cfg &c, const void *x, const moe_params &p, const State &st, const EpSrcBwd &b,
                   const moe_grads &gr, const DeviceInfo &dev, cudaStream_t stream)
{
    t_launches = 0;
    t_pdl = false;
    const Shapes s = shapes(c);
    const int n_parts = c.I % 256 == 0 ? c.I / 256 : c.I / 128;
    MOK_TRY(launch_k(slot_grad_kernel, dim3(blocks_for(s.T, 256)), dim3(256), 0, stream, "slot_grad_kernel",
                     static_cast<const float *>(b.gpart), n_parts, static_cast<const int *>(st.inv_perm),
                     static_cast<const float *>(st.topk_w), static_cast<const float *>(st.topk_p), b.dl, c.T,
                     c.top_k, c.score_fn, c.routed_scale));
    MOK_TRY(launch_k(drouter_partial_kernel, dim3(static_cast<unsigned>(s.max_chunks), c.H / 256), dim3(256), 0, stream,
                     "drouter_partial_kernel", static_cast<const __nv_bfloat16 *>(x), static_cast<const float *>(b.dl),
                     static_cast<const int *>(st.offsets), static_cast<const int *>(st.chunk_start),
                     static_cast<const int *>(st.perm), b.partial, c.H, c.E, c.top_k, kChunkRows));
    MOK_TRY(launch_k(drouter_reduce_kernel, dim3(blocks_for(s.E * s.H, 256)), dim3(256), 0, stream,
                     "drouter_reduce_kernel", static_cast<const float *>(b.partial),
                     static_cast<const int *>(st.chunk_start), gr.drouter_w, c.H, c.E));
    return launch_k(dx_combine_kernel, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0, stream,
                    "dx_combine_kernel", static_cast<const float *>(b.dxs), static_cast<const float *>(b.dl),
                    static_cast<const int *>(st.topk_idx), p.router_w, static_cast<__nv_bfloat16 *>(gr.dx), c.T, c.H,
                    c.top_k, c.n_shared);
}

PFN_cuMemGetAddressRange_v3020 g_addr_range = nullptr;

}  // namespace
}  // namespace mok

using namespace mok;

extern "C" {

int moe_workspace_size(const moe_cfg *cfg, size_t *ctx_bytes, size_t *fwd_scratch_bytes, size_t *bwd_scratch_bytes)
{
    MOK_TRY(check_cfg(cfg));
    if (ctx_bytes) *ctx_bytes = carve_state(*cfg, nullptr, true).bytes;
    if (fwd_scratch_bytes) *fwd_scratch_bytes = carve_state(*cfg, nullptr, false).bytes;
    if (bwd_scratch_bytes) *bwd_scratch_bytes = carve_bwd(*cfg, nullptr).bytes;
    return MOK_OK;
}

int moe_fwd(const moe_cfg *cfg, const void *x, const moe_params *params, void *y, const moe_routing *routing,
            void *ctx, size_t ctx_bytes, int save_for_backward, void *scratch, size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    MOK_TRY(check_params(*cfg, params));
    if (!x || !y || !aligned16(x) || !aligned16(y)) return MOK_ERR_INVALID;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    const bool training = save_for_backward != 0;
    void *buf = training ? ctx : scratch;
    const size_t have = training ? ctx_bytes : scratch_bytes;
    const State need = carve_state(*cfg, nullptr, training);
    if (!buf || have < need.bytes) return MOK_ERR_WORKSPACE;
    if (!aligned16(buf)) return MOK_ERR_INVALID;
    const State st = carve_state(*cfg, buf, training);
    return forward(*cfg, x, *params, y, routing, st, *dev, training, static_cast<cudaStream_t>(stream));
}

int moe_bwd(const moe_cfg *cfg, const void *x, const void *dy, const moe_params *params, const void *ctx,
            size_t ctx_bytes, const moe_grads *grads, void *scratch, size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    MOK_TRY(check_params(*cfg, params));
    if (cfg->dtype == MOK_DTYPE_MXFP8) {
        const moe_params &q = *params;
        if (!q.wt_gate_up || !q.wt_down || !q.st_gate_up || !q.st_down ||
            (cfg->n_shared > 0 && (!q.wst_gate_up || !q.wst_down || !q.sst_gate_up || !q.sst_down)))
            return fail(MOK_ERR_INVALID, "moe_bwd (MXFP8): the transposed weight copies wt_* / st_* are missing");
        const void *w[] = {q.wt_gate_up, q.wt_down, q.wst_gate_up, q.wst_down};
        for (const void *v : w)
            if (v && !aligned16(v)) return MOK_ERR_INVALID;
        if (cfg->I % 256) return fail(MOK_ERR_UNSUPPORTED, "moe_bwd (MXFP8): I must be a multiple of 256");
    }
    if (!x || !dy || !grads || !grads->dx || !grads->dw_gate_up || !grads->dw_down || !grads->drouter_w)
        return MOK_ERR_INVALID;
    if (cfg->n_shared > 0 && (!grads->dws_gate_up || !grads->dws_down)) return MOK_ERR_INVALID;
    const void *ptrs[] = {x, dy, grads->dx, grads->dw_gate_up, grads->dw_down, grads->drouter_w,
                          grads->dws_gate_up, grads->dws_down};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return MOK_ERR_INVALID;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    if (!ctx || ctx_bytes < carve_state(*cfg, nullptr, true).bytes) return MOK_ERR_WORKSPACE;
    if (!scratch || scratch_bytes < carve_bwd(*cfg, nullptr).bytes) return MOK_ERR_WORKSPACE;
    if (!aligned16(ctx) || !aligned16(scratch)) return MOK_ERR_INVALID;
    const State st = carve_state(*cfg, const_cast<void *>(ctx), true);
    const BwdScratch bs = carve_bwd(*cfg, scratch);
    return backward(*cfg, x, dy, *params, st, *grads, bs, *dev, static_cast<cudaStream_t>(stream));
}

int moe_host_scratch_size(const moe_cfg *cfg, int backward, size_t *bytes)
{
    MOK_TRY(check_cfg(cfg));
    const size_t io = align_up(static_cast<size_t>(cfg->T) * cfg->H * 2, 256);
    size_t inner = backward ? carve_bwd(*cfg, nullptr).bytes : carve_state(*cfg, nullptr, false).bytes;
    if (bytes) *bytes = (backward == 3 ? 6 : backward == 2 ? 4 : backward ? 3 : 2) * io + inner;
    return MOK_OK;
}

int moe_fwd_host(const moe_cfg *cfg, const void *x_host, const moe_params *params, void *y_host, void *ctx,
                 size_t ctx_bytes, int save_for_backward, void *scratch, size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    if (!x_host || !y_host || !scratch) return MOK_ERR_INVALID;
    size_t need = 0;
    moe_host_scratch_size(cfg, 0, &need);
    if (scratch_bytes < need) return MOK_ERR_WORKSPACE;
    const size_t io = align_up(static_cast<size_t>(cfg->T) * cfg->H * 2, 256);
    char *s = static_cast<char *>(scratch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t nb = static_cast<size_t>(cfg->T) * cfg->H * 2;
    if (const cudaError_t e_ = cudaMemcpyAsync(s, x_host, nb, cudaMemcpyHostToDevice, st); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync", e_);
    MOK_TRY(moe_fwd(cfg, s, params, s + io, nullptr, ctx, ctx_bytes, save_for_backward, s + 2 * io,
                    scratch_bytes - 2 * io, stream));
    if (const cudaError_t e_ = cudaMemcpyAsync(y_host, s + io, nb, cudaMemcpyDeviceToHost, st); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync", e_);
    if (const cudaError_t e_ = cudaStreamSynchronize(st); e_ != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize", e_);
    return MOK_OK;
}

int moe_bwd_host(const moe_cfg *cfg, const void *x_host, const void *dy_host, const moe_params *params,
                 const void *ctx, size_t ctx_bytes, void *dx_host, const moe_grads *grads, void *scratch,
                 size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    if (!dy_host || !dx_host || !scratch || !grads) return MOK_ERR_INVALID;
    size_t need = 0;
    moe_host_scratch_size(cfg, 1, &need);
    if (scratch_bytes < need) return MOK_ERR_WORKSPACE;
    const size_t io = align_up(static_cast<size_t>(cfg->T) * cfg->H * 2, 256);
    char *s = static_cast<char *>(scratch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t nb = static_cast<size_t>(cfg->T) * cfg->H * 2;
    if (x_host)                 // NULL: x is still in the scratch from the preceding moe_fwd_host
        if (const cudaError_t e_ = cudaMemcpyAsync(s, x_host, nb, cudaMemcpyHostToDevice, st); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync", e_);
    if (const cudaError_t e_ = cudaMemcpyAsync(s + io, dy_host, nb, cudaMemcpyHostToDevice, st); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync", e_);
    moe_grads g = *grads;
    g.dx = s + 2 * io;
    MOK_TRY(moe_bwd(cfg, s, s + io, params, ctx, ctx_bytes, &g, s + 3 * io, scratch_bytes - 3 * io, stream));
    if (const cudaError_t e_ = cudaMemcpyAsync(dx_host, s + 2 * io, nb, cudaMemcpyDeviceToHost, st); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyAsync", e_);
    if (const cudaError_t e_ = cudaStreamSynchronize(st); e_ != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize", e_);
    return MOK_OK;
}

namespace {
// The second stream and the events of moe_step_host, per host thread and device.
struct StepStreams {
    int device = -1;
    cudaStream_t side = nullptr;
    cudaEvent_t start = nullptr, dy_in = nullptr, y_ready = nullptr, y_out = nullptr;
};
thread_local StepStreams t_step;

// Pipelined host steps (moe_step_host_async): an upload and a download stream per
// host thread and device, the events that order them with the caller's stream,
// and which host x each of the two device x slots holds.
struct PipeStreams {
    int device = -1;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t fwd_done = nullptr, bwd_done = nullptr, dy_in = nullptr, y_out = nullptr;
    cudaEvent_t x_ready[2] = {nullptr, nullptr}, dx_out[2] = {nullptr, nullptr};
    const void *scratch = nullptr;      // the scratch buffer of the calls in flight
    const void *slot_x[2] = {nullptr, nullptr};   // host x uploaded (or on its way) into each slot
    unsigned long long calls = 0;
};
thread_local PipeStreams t_pipe;

int pipe_streams(PipeStreams *&ps)
{
    int dev = 0;
    if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return fail(MOK_ERR_DEVICE, "cudaGetDevice", e);
    ps = &t_pipe;
    if (ps->device == dev) return MOK_OK;
    if (ps->up) {                   // another device: release the old handles first
        cudaStreamSynchronize(ps->up);
        cudaStreamSynchronize(ps->down);
        cudaStreamDestroy(ps->up);
        cudaStreamDestroy(ps->down);
        cudaEvent_t evs[] = {ps->fwd_done, ps->bwd_done, ps->dy_in, ps->y_out, ps->x_ready[0], ps->x_ready[1],
                             ps->dx_out[0], ps->dx_out[1]};
        for (cudaEvent_t ev : evs) cudaEventDestroy(ev);
        *ps = PipeStreams{};
    }
    if (const cudaError_t e = cudaStreamCreateWithFlags(&ps->up, cudaStreamNonBlocking); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaStreamCreateWithFlags", e);
    if (const cudaError_t e = cudaStreamCreateWithFlags(&ps->down, cudaStreamNonBlocking); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaStreamCreateWithFlags", e);
    cudaEvent_t *evs[] = {&ps->fwd_done, &ps->bwd_done, &ps->dy_in, &ps->y_out, &ps->x_ready[0], &ps->x_ready[1],
                          &ps->dx_out[0], &ps->dx_out[1]};
    for (cudaEvent_t *ev : evs)
        if (const cudaError_t e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming); e != cudaSuccess)
            return fail(MOK_ERR_LAUNCH, "cudaEventCreateWithFlags", e);
    ps->device = dev;
    return MOK_OK;
}

int step_streams(StepStreams *&ss)
{
    int dev = 0;
    if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return fail(MOK_ERR_DEVICE, "cudaGetDevice", e);
    ss = &t_step;
    if (ss->device == dev) return MOK_OK;
    if (ss->side) {                 // another device: release the old handles first
        cudaStreamDestroy(ss->side);
        cudaEventDestroy(ss->start);
        cudaEventDestroy(ss->dy_in);
        cudaEventDestroy(ss->y_ready);
        cudaEventDestroy(ss->y_out);
        *ss = StepStreams{};
    }
    if (const cudaError_t e = cudaStreamCreateWithFlags(&ss->side, cudaStreamNonBlocking); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaStreamCreateWithFlags", e);
    cudaEvent_t *evs[] = {&ss->start, &ss->dy_in, &ss->y_ready, &ss->y_out};
    for (cudaEvent_t *ev : evs)
        if (const cudaError_t e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming); e != cudaSuccess)
            return fail(MOK_ERR_LAUNCH, "cudaEventCreateWithFlags", e);
    ss->device = dev;
    return MOK_OK;
}
}  // namespace

int moe_step_host(const moe_cfg *cfg, const void *x_host, const void *dy_host, const moe_params *params,
                  void *y_host, void *dx_host, void *ctx, size_t ctx_bytes, const moe_grads *grads, void *scratch,
                  size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    if (!x_host || !dy_host || !y_host || !dx_host || !scratch || !grads) return MOK_ERR_INVALID;
    size_t need = 0;
    moe_host_scratch_size(cfg, 2, &need);
    if (scratch_bytes < need) return MOK_ERR_WORKSPACE;
    if (!device_info()) return MOK_ERR_DEVICE;
    StepStreams *ss = nullptr;
    MOK_TRY(step_streams(ss));
    const size_t io = align_up(static_cast<size_t>(cfg->T) * cfg->H * 2, 256);
    const size_t nb = static_cast<size_t>(cfg->T) * cfg->H * 2;
    char *s = static_cast<char *>(scratch);
    char *x = s, *y = s + io, *dy = s + 2 * io, *dx = s + 3 * io, *inner = s + 4 * io;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    int rc = MOK_OK;
#define STEP_CUDA(call, what)                                      \
    if ((e = (call)) != cudaSuccess) {                             \
        rc = fail(MOK_ERR_LAUNCH, what, e);                        \
        goto done;                                                 \
    }
    // the side stream starts after everything already enqueued on `stream` (which may
    // still read this scratch buffer)
    STEP_CUDA(cudaEventRecord(ss->start, st), "cudaEventRecord");
    STEP_CUDA(cudaStreamWaitEvent(ss->side, ss->start, 0), "cudaStreamWaitEvent");
    STEP_CUDA(cudaMemcpyAsync(dy, dy_host, nb, cudaMemcpyHostToDevice, ss->side), "cudaMemcpyAsync(dy)");
    STEP_CUDA(cudaEventRecord(ss->dy_in, ss->side), "cudaEventRecord");
    STEP_CUDA(cudaMemcpyAsync(x, x_host, nb, cudaMemcpyHostToDevice, st), "cudaMemcpyAsync(x)");
    if ((rc = moe_fwd(cfg, x, params, y, nullptr, ctx, ctx_bytes, 1, nullptr, 0, stream)) != MOK_OK) goto done;
    // y leaves on the side stream while the backward runs
    STEP_CUDA(cudaEventRecord(ss->y_ready, st), "cudaEventRecord");
    STEP_CUDA(cudaStreamWaitEvent(ss->side, ss->y_ready, 0), "cudaStreamWaitEvent");
    STEP_CUDA(cudaMemcpyAsync(y_host, y, nb, cudaMemcpyDeviceToHost, ss->side), "cudaMemcpyAsync(y)");
    STEP_CUDA(cudaEventRecord(ss->y_out, ss->side), "cudaEventRecord");
    STEP_CUDA(cudaStreamWaitEvent(st, ss->dy_in, 0), "cudaStreamWaitEvent");
    {
        moe_grads g = *grads;
        g.dx = dx;
        if ((rc = moe_bwd(cfg, x, dy, params, ctx, ctx_bytes, &g, inner, scratch_bytes - 4 * io, stream)) != MOK_OK)
            goto done;
    }
    STEP_CUDA(cudaMemcpyAsync(dx_host, dx, nb, cudaMemcpyDeviceToHost, st), "cudaMemcpyAsync(dx)");
    STEP_CUDA(cudaStreamWaitEvent(st, ss->y_out, 0), "cudaStreamWaitEvent");
#undef STEP_CUDA
done:
    // both streams drain before the call returns, on success and on failure
    if (const cudaError_t e2 = cudaStreamSynchronize(ss->side); e2 != cudaSuccess && rc == MOK_OK)
        rc = fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize(side)", e2);
    if (const cudaError_t e2 = cudaStreamSynchronize(st); e2 != cudaSuccess && rc == MOK_OK)
        rc = fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize", e2);
    return rc;
}

int moe_step_host_async(const moe_cfg *cfg, const void *x_host, const void *x_next_host, const void *dy_host,
                        const moe_params *params, void *y_host, void *dx_host, void *ctx, size_t ctx_bytes,
                        const moe_grads *grads, void *scratch, size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    if (!x_host || !dy_host || !y_host || !dx_host || !scratch || !grads) return MOK_ERR_INVALID;
    size_t need = 0;
    moe_host_scratch_size(cfg, 3, &need);
    if (scratch_bytes < need) return MOK_ERR_WORKSPACE;
    if (!device_info()) return MOK_ERR_DEVICE;
    PipeStreams *ps = nullptr;
    MOK_TRY(pipe_streams(ps));
    if (ps->scratch != scratch) {       // a new sequence: nothing of this buffer is prefetched
        ps->scratch = scratch;
        ps->slot_x[0] = ps->slot_x[1] = nullptr;
        ps->calls = 0;
    }
    const int p = static_cast<int>(ps->calls & 1u);
    const size_t io = align_up(static_cast<size_t>(cfg->T) * cfg->H * 2, 256);
    const size_t nb = static_cast<size_t>(cfg->T) * cfg->H * 2;
    char *s = static_cast<char *>(scratch);
    char *xs[2] = {s, s + io}, *y = s + 2 * io, *dy = s + 3 * io, *dxs[2] = {s + 4 * io, s + 5 * io};
    char *inner = s + 6 * io;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    int rc = MOK_OK;
#define PIPE_CUDA(call, what)                                      \
    if ((e = (call)) != cudaSuccess) {                             \
        rc = fail(MOK_ERR_LAUNCH, what, e);                        \
        goto fail_sync;                                            \
    }
    // x of this step in slot p: prefetched by the previous call, or uploaded now (after
    // any prefetch still landing in that slot)
    PIPE_CUDA(cudaStreamWaitEvent(st, ps->x_ready[p], 0), "cudaStreamWaitEvent");
    if (ps->slot_x[p] != x_host) {
        PIPE_CUDA(cudaMemcpyAsync(xs[p], x_host, nb, cudaMemcpyHostToDevice, st), "cudaMemcpyAsync(x)");
        ps->slot_x[p] = x_host;
    }
    // dy on the upload stream once the previous step's backward has read the buffer
    PIPE_CUDA(cudaStreamWaitEvent(ps->up, ps->bwd_done, 0), "cudaStreamWaitEvent");
    PIPE_CUDA(cudaMemcpyAsync(dy, dy_host, nb, cudaMemcpyHostToDevice, ps->up), "cudaMemcpyAsync(dy)");
    PIPE_CUDA(cudaEventRecord(ps->dy_in, ps->up), "cudaEventRecord");
    // the forward writes y once the previous step's y has left
    PIPE_CUDA(cudaStreamWaitEvent(st, ps->y_out, 0), "cudaStreamWaitEvent");
    if ((rc = moe_fwd(cfg, xs[p], params, y, nullptr, ctx, ctx_bytes, 1, nullptr, 0, stream)) != MOK_OK)
        goto fail_sync;
    PIPE_CUDA(cudaEventRecord(ps->fwd_done, st), "cudaEventRecord");
    PIPE_CUDA(cudaStreamWaitEvent(ps->down, ps->fwd_done, 0), "cudaStreamWaitEvent");
    PIPE_CUDA(cudaMemcpyAsync(y_host, y, nb, cudaMemcpyDeviceToHost, ps->down), "cudaMemcpyAsync(y)");
    PIPE_CUDA(cudaEventRecord(ps->y_out, ps->down), "cudaEventRecord");
    // the next step's x into the other slot while this step's backward runs (its last
    // reader, the previous step, is done: the upload stream waited for it above)
    if (x_next_host) {
        PIPE_CUDA(cudaMemcpyAsync(xs[1 - p], x_next_host, nb, cudaMemcpyHostToDevice, ps->up),
                  "cudaMemcpyAsync(next x)");
        PIPE_CUDA(cudaEventRecord(ps->x_ready[1 - p], ps->up), "cudaEventRecord");
        ps->slot_x[1 - p] = x_next_host;
    } else {
        ps->slot_x[1 - p] = nullptr;
    }
    // the backward writes dx into slot p once the download of two steps ago has read it
    PIPE_CUDA(cudaStreamWaitEvent(st, ps->dy_in, 0), "cudaStreamWaitEvent");
    PIPE_CUDA(cudaStreamWaitEvent(st, ps->dx_out[p], 0), "cudaStreamWaitEvent");
    {
        moe_grads g = *grads;
        g.dx = dxs[p];
        if ((rc = moe_bwd(cfg, xs[p], dy, params, ctx, ctx_bytes, &g, inner, scratch_bytes - 6 * io, stream)) !=
            MOK_OK)
            goto fail_sync;
    }
    PIPE_CUDA(cudaEventRecord(ps->bwd_done, st), "cudaEventRecord");
    PIPE_CUDA(cudaStreamWaitEvent(ps->down, ps->bwd_done, 0), "cudaStreamWaitEvent");
    PIPE_CUDA(cudaMemcpyAsync(dx_host, dxs[p], nb, cudaMemcpyDeviceToHost, ps->down), "cudaMemcpyAsync(dx)");
    PIPE_CUDA(cudaEventRecord(ps->dx_out[p], ps->down), "cudaEventRecord");
#undef PIPE_CUDA
    ++ps->calls;
    return MOK_OK;
fail_sync:
    // a failed step leaves nothing in flight: every stream of the sequence drains
    cudaStreamSynchronize(ps->up);
    cudaStreamSynchronize(ps->down);
    cudaStreamSynchronize(st);
    ps->scratch = nullptr;
    return rc;
}

int moe_step_host_sync(void *stream)
{
    PipeStreams *ps = nullptr;
    MOK_TRY(pipe_streams(ps));
    int rc = MOK_OK;
    cudaStream_t ss[] = {ps->up, ps->down, static_cast<cudaStream_t>(stream)};
    for (cudaStream_t s2 : ss)
        if (const cudaError_t e = cudaStreamSynchronize(s2); e != cudaSuccess && rc == MOK_OK)
            rc = fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize", e);
    return rc;
}

static int quantize(const void *src, int64_t rows, int64_t K, void *q, void *scales, bool packed, void *stream)
{
    if (!src || !q || !scales || rows < 0 || K <= 0 || K % 32) return MOK_ERR_INVALID;
    if (packed && (rows % 128 || K % 128)) return fail(MOK_ERR_INVALID, "moe_quantize_mxfp8_weights: rows and K must be multiples of 128");
    if (!aligned16(src) || !aligned16(q)) return MOK_ERR_INVALID;
    if (!device_info()) return MOK_ERR_DEVICE;
    const long long nb = rows * (K / 32);
    if (nb == 0) return MOK_OK;
    quantize_mxfp8_kernel<<<blocks_for(nb, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(src), nb, static_cast<uint8_t *>(q), static_cast<uint8_t *>(scales), K / 32,
        packed ? rows / 128 : 0, static_cast<__nv_bfloat16 *>(nullptr));
    if (const cudaError_t e_ = cudaGetLastError(); e_ != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "quantize_mxfp8_kernel launch", e_);
    return MOK_OK;
}

int moe_quantize_mxfp8(const void *src, int64_t rows, int64_t K, void *q, void *scales, void *stream)
{
    return quantize(src, rows, K, q, scales, false, stream);
}

int moe_quantize_mxfp8_weights(const void *src, int64_t rows, int64_t K, void *q, void *scales, void *stream)
{
    return quantize(src, rows, K, q, scales, true, stream);
}

int moe_quantize_mxfp8_weights_t(const void *src, int64_t batch, int64_t R, int64_t C, void *q, void *scales,
                                 void *stream)
{
    if (!src || !q || !scales || batch < 0 || R <= 0 || C <= 0) return MOK_ERR_INVALID;
    if (R % 128 || C % 32 || (batch * C) % 128)
        return fail(MOK_ERR_INVALID, "moe_quantize_mxfp8_weights_t: R and batch*C must be multiples of 128, C of 32");
    if (!aligned16(src) || !aligned16(q)) return MOK_ERR_INVALID;
    if (!device_info()) return MOK_ERR_DEVICE;
    const long long n = batch * C * (R / 32);
    if (n == 0) return MOK_OK;
    quantize_mxfp8_t_kernel<<<blocks_for(n, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(src), batch, R, C, static_cast<uint8_t *>(q), static_cast<uint8_t *>(scales));
    if (const cudaError_t e_ = cudaGetLastError(); e_ != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "quantize_mxfp8_t_kernel launch", e_);
    return MOK_OK;
}

int moe_quantize_mxfp8_weights_both(const void *src, int64_t batch, int64_t R, int64_t C, void *q, void *scales,
                                    void *qt, void *scales_t, void *stream)
{
    if (!src || !q || !scales || !qt || !scales_t || batch < 0 || R <= 0 || C <= 0) return MOK_ERR_INVALID;
    if (R % 128 || C % 256)
        return fail(MOK_ERR_INVALID, "moe_quantize_mxfp8_weights_both: R must be a multiple of 128, C of 256");
    if (!aligned16(src) || !aligned16(q) || !aligned16(qt)) return MOK_ERR_INVALID;
    if (!device_info()) return MOK_ERR_DEVICE;
    const long long n = batch * (R / 32) * (C / kQuantBothCols);
    if (n == 0) return MOK_OK;
    quantize_mxfp8_both_kernel<<<static_cast<unsigned>(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(src), batch, R, C, static_cast<uint8_t *>(q), static_cast<uint8_t *>(scales),
        static_cast<uint8_t *>(qt), static_cast<uint8_t *>(scales_t));
    if (const cudaError_t e_ = cudaGetLastError(); e_ != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "quantize_mxfp8_both_kernel launch", e_);
    return MOK_OK;
}

int moe_trace_events(void *const *fwd_events, int n_fwd, void *const *bwd_events, int n_bwd)
{
    if (n_fwd < 0 || n_bwd < 0) return MOK_ERR_INVALID;
    if (n_fwd > 0 && (n_fwd < MOK_FWD_PHASES + 1 || !fwd_events)) return MOK_ERR_INVALID;
    if (n_bwd > 0 && (n_bwd < MOK_BWD_PHASES + 1 || !bwd_events)) return MOK_ERR_INVALID;
    for (int i = 0; i < (n_fwd > 0 ? MOK_FWD_PHASES + 1 : 0); ++i)
        if (!fwd_events[i]) return fail(MOK_ERR_INVALID, "moe_trace_events: NULL event handle");
    for (int i = 0; i < (n_bwd > 0 ? MOK_BWD_PHASES + 1 : 0); ++i)
        if (!bwd_events[i]) return fail(MOK_ERR_INVALID, "moe_trace_events: NULL event handle");
    t_fwd_on = n_fwd > 0;
    t_bwd_on = n_bwd > 0;
    for (int i = 0; t_fwd_on && i <= MOK_FWD_PHASES; ++i) t_fwd_ev[i] = static_cast<cudaEvent_t>(fwd_events[i]);
    for (int i = 0; t_bwd_on && i <= MOK_BWD_PHASES; ++i) t_bwd_ev[i] = static_cast<cudaEvent_t>(bwd_events[i]);
    return MOK_OK;
}

int moe_status(void *stream, int32_t *device_status)
{
    if (!device_status) return MOK_ERR_INVALID;
    if (!device_info()) return MOK_ERR_DEVICE;
    if (const cudaError_t e_ = cudaStreamSynchronize(static_cast<cudaStream_t>(stream)); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaStreamSynchronize", e_);
    int v = 0;
    if (const cudaError_t e_ = cudaMemcpyFromSymbol(&v, g_status, sizeof(int)); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyFromSymbol", e_);
    const int zero = 0;
    if (const cudaError_t e_ = cudaMemcpyToSymbol(g_status, &zero, sizeof(int)); e_ != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaMemcpyToSymbol", e_);
    *device_status = v;
    return MOK_OK;
}

int moe_fwd_static(const moe_cfg *cfg, const void *x, const moe_params *params, void *y, void *stream)
{
    MOK_TRY(check_cfg(cfg));
    MOK_TRY(check_params(*cfg, params));
    if (!x || !y || !aligned16(x) || !aligned16(y)) return fail(MOK_ERR_INVALID, "moe_fwd_static: x or y");
    const size_t need = carve_state(*cfg, nullptr, false).bytes;
    if (need > MOK_STATIC_SCRATCH_BYTES) {
        snprintf(t_last_error, sizeof(t_last_error),
                 "moe_fwd_static: this shape needs %zu bytes of scratch; the static scratch holds %u bytes",
                 need, MOK_STATIC_SCRATCH_BYTES);
        return MOK_ERR_WORKSPACE;
    }
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    // once per device, with that device current: the array's device address
    static void *s_static_ptr[kMaxDevices] = {};
    int d = 0;
    if (const cudaError_t e = cudaGetDevice(&d); e != cudaSuccess) return fail(MOK_ERR_LAUNCH, "cudaGetDevice", e);
    void *ptr = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!s_static_ptr[d]) {
            void *p = nullptr;
            if (const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch); e != cudaSuccess)
                return fail(MOK_ERR_LAUNCH, "cudaGetSymbolAddress(static scratch)", e);
            s_static_ptr[d] = p;
        }
        ptr = s_static_ptr[d];
    }
    const State st = carve_state(*cfg, ptr, false);
    return forward(*cfg, x, *params, y, nullptr, st, *dev, false, static_cast<cudaStream_t>(stream));
}

int moe_saved_tensor(const moe_cfg *cfg, int save_for_backward, int which, size_t *offset, size_t *bytes)
{
    MOK_TRY(check_cfg(cfg));
    const bool training = save_for_backward != 0;
    // carve over a stand-in base address: only the differences are used
    char *const base = reinterpret_cast<char *>(uintptr_t(1) << 40);
    const State st = carve_state(*cfg, base, training);
    const Shapes s = shapes(*cfg);
    const void *p = nullptr;
    size_t n = 0;
    switch (which) {
    case MOK_SAVED_H: p = st.h; n = s.R * s.I * 2; break;
    case MOK_SAVED_HQ: p = st.hq; n = s.R * s.I; break;
    case MOK_SAVED_HS: p = st.hs; n = s.R * s.I / 32; break;
    case MOK_SAVED_GU: p = st.gu; n = s.R * 2 * s.I * 2; break;
    case MOK_SAVED_HW: p = st.hw; n = s.R * s.I * 2; break;
    case MOK_SAVED_ROW_TOKEN: p = st.row_token; n = s.R * 4; break;
    case MOK_SAVED_ROW_W: p = st.row_w; n = s.R * 4; break;
    default: return MOK_ERR_INVALID;
    }
    if (!p) return MOK_ERR_UNSUPPORTED;
    if (offset) *offset = static_cast<size_t>(static_cast<const char *>(p) - base);
    if (bytes) *bytes = n;
    return MOK_OK;
}

int moe_ep_size(const moe_cfg *cfg, int32_t world, int32_t training, size_t *state_bytes, size_t *scratch_bytes,
                size_t *bwd_bytes)
{
    MOK_TRY(check_ep(cfg, world, 0));
    if (training && cfg->dtype == MOK_DTYPE_MXFP8 && cfg->I % 256) return MOK_ERR_UNSUPPORTED;
    if (state_bytes) *state_bytes = carve_state(*cfg, nullptr, false).bytes;
    if (scratch_bytes) *scratch_bytes = carve_ep(*cfg, world, training != 0, nullptr).bytes;
    if (bwd_bytes) *bwd_bytes = carve_ep_src_bwd(*cfg, nullptr).bytes;
    return MOK_OK;
}

int moe_ep_route(const moe_cfg *cfg, int32_t world, int32_t rank, const void *x, const moe_params *params,
                 void *state, size_t state_bytes, void *stream)
{
    MOK_TRY(check_ep(cfg, world, rank));
    if (!params || !params->router_w || !aligned16(params->router_w)) return MOK_ERR_INVALID;
    if (!x || !aligned16(x) || !state || !aligned16(state)) return MOK_ERR_INVALID;
    if (state_bytes < carve_state(*cfg, nullptr, false).bytes) return MOK_ERR_WORKSPACE;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    return ep_route(*cfg, x, *params, carve_state(*cfg, state, false), *dev, static_cast<cudaStream_t>(stream));
}

int moe_ep_experts(const moe_cfg *cfg, int32_t world, int32_t rank, int32_t training, const void *const *x_ranks,
                   void *const *state_ranks, const moe_params *params, void *scratch, size_t scratch_bytes,
                   void *stream)
{
    MOK_TRY(check_ep(cfg, world, rank));
    if (training && cfg->dtype == MOK_DTYPE_MXFP8 && cfg->I % 256) return MOK_ERR_UNSUPPORTED;
    if (!params || !params->w_gate_up || !params->w_down || !x_ranks || !state_ranks) return MOK_ERR_INVALID;
    if (cfg->n_shared > 0 && (!params->ws_gate_up || !params->ws_down)) return MOK_ERR_INVALID;
    if (cfg->dtype == MOK_DTYPE_MXFP8 &&
        (!params->s_gate_up || !params->s_down || (cfg->n_shared > 0 && (!params->ss_gate_up || !params->ss_down))))
        return MOK_ERR_INVALID;
    const void *w[] = {params->w_gate_up, params->w_down, params->ws_gate_up, params->ws_down};
    for (const void *q : w)
        if (q && !aligned16(q)) return MOK_ERR_INVALID;
    for (int r = 0; r < world; ++r)
        if (!x_ranks[r] || !state_ranks[r] || !aligned16(x_ranks[r]) || !aligned16(state_ranks[r]))
            return MOK_ERR_INVALID;
    if (!scratch || !aligned16(scratch)) return MOK_ERR_INVALID;
    const EpScratch need = carve_ep(*cfg, world, training != 0, nullptr);
    if (scratch_bytes < need.bytes) return MOK_ERR_WORKSPACE;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    return ep_experts(*cfg, world, rank, training != 0, x_ranks, state_ranks, *params,
                      carve_ep(*cfg, world, training != 0, scratch), *dev, static_cast<cudaStream_t>(stream));
}

int moe_ep_bwd_experts(const moe_cfg *cfg, int32_t world, int32_t rank, const void *const *dy_ranks,
                       void *const *bwd_ranks, const moe_params *params, const moe_grads *grads, void *scratch,
                       size_t scratch_bytes, void *stream)
{
    MOK_TRY(check_ep(cfg, world, rank));
    if (cfg->dtype == MOK_DTYPE_MXFP8 && cfg->I % 256) return MOK_ERR_UNSUPPORTED;
    if (!params || !params->w_gate_up || !params->w_down || !dy_ranks || !bwd_ranks || !grads) return MOK_ERR_INVALID;
    if (cfg->dtype == MOK_DTYPE_MXFP8) {
        // the transposed weight copies of the data gradients (moe_quantize_mxfp8_weights_t of the rank's slice)
        const moe_params &q = *params;
        if (!q.wt_gate_up || !q.wt_down || !q.st_gate_up || !q.st_down ||
            (cfg->n_shared > 0 && (!q.wst_gate_up || !q.wst_down || !q.sst_gate_up || !q.sst_down)))
            return MOK_ERR_INVALID;
    }
    if (cfg->n_shared > 0 && (!params->ws_gate_up || !params->ws_down || !grads->dws_gate_up || !grads->dws_down))
        return MOK_ERR_INVALID;
    const void *w[] = {params->w_gate_up, params->w_down, params->ws_gate_up, params->ws_down, grads->dw_gate_up,
                       grads->dw_down, grads->dws_gate_up, grads->dws_down};
    for (const void *q : w)
        if (q && !aligned16(q)) return MOK_ERR_INVALID;
    if (!grads->dw_gate_up || !grads->dw_down) return MOK_ERR_INVALID;
    for (int r = 0; r < world; ++r)
        if (!dy_ranks[r] || !bwd_ranks[r] || !aligned16(dy_ranks[r]) || !aligned16(bwd_ranks[r]))
            return MOK_ERR_INVALID;
    if (!scratch || !aligned16(scratch)) return MOK_ERR_INVALID;
    if (scratch_bytes < carve_ep(*cfg, world, true, nullptr).bytes) return MOK_ERR_WORKSPACE;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    return ep_bwd_experts(*cfg, world, rank, dy_ranks, bwd_ranks, *params, *grads, carve_ep(*cfg, world, true, scratch),
                          *dev, static_cast<cudaStream_t>(stream));
}

int moe_ep_bwd_combine(const moe_cfg *cfg, int32_t world, int32_t rank, const void *x, const moe_params *params,
                       const void *state, void *bwd, size_t bwd_bytes, const moe_grads *grads, void *stream)
{
    MOK_TRY(check_ep(cfg, world, rank));
    if (!params || !params->router_w || !aligned16(params->router_w) || !grads || !grads->dx || !grads->drouter_w)
        return MOK_ERR_INVALID;
    if (!aligned16(grads->dx) || !aligned16(grads->drouter_w)) return MOK_ERR_INVALID;
    if (!x || !aligned16(x) || !state || !aligned16(state) || !bwd || !aligned16(bwd)) return MOK_ERR_INVALID;
    if (bwd_bytes < carve_ep_src_bwd(*cfg, nullptr).bytes) return MOK_ERR_WORKSPACE;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    return ep_bwd_combine(*cfg, x, *params, carve_state(*cfg, const_cast<void *>(state), false),
                          carve_ep_src_bwd(*cfg, bwd), *grads, *dev, static_cast<cudaStream_t>(stream));
}

int moe_ep_combine(const moe_cfg *cfg, int32_t world, int32_t rank, const void *state, void *y, void *stream)
{
    MOK_TRY(check_ep(cfg, world, rank));
    if (!state || !aligned16(state) || !y || !aligned16(y)) return MOK_ERR_INVALID;
    const DeviceInfo *dev = device_info();
    if (!dev) return MOK_ERR_DEVICE;
    t_launches = 0;
    t_pdl = false;
    const State st = carve_state(*cfg, const_cast<void *>(state), false);
    const Shapes s = shapes(*cfg);
    if (cfg->dtype == MOK_DTYPE_MXFP8)       // the MXFP8 forward's slot rows are bf16
        return launch_k(combine_kernel<__nv_bfloat16>, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0,
                        static_cast<cudaStream_t>(stream), "combine_kernel",
                        reinterpret_cast<const __nv_bfloat16 *>(st.O), static_cast<const float *>(st.topk_w),
                        static_cast<__nv_bfloat16 *>(y), cfg->T, cfg->H, cfg->top_k, cfg->n_shared);
    return launch_k(combine_kernel<float>, dim3(blocks_for(s.T * s.H / 8, 256)), dim3(256), 0,
                    static_cast<cudaStream_t>(stream), "combine_kernel", static_cast<const float *>(st.O),
                    static_cast<const float *>(st.topk_w), static_cast<__nv_bfloat16 *>(y), cfg->T, cfg->H,
                    cfg->top_k, cfg->n_shared);
}

static int ep_alloc_base(const void *dev_ptr, char **base)
{
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_addr_range) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                g_addr_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
        }
    }
    if (!g_addr_range) return fail(MOK_ERR_DEVICE, "cuMemGetAddressRange not available");
    CUdeviceptr b = 0;
    size_t n = 0;
    if (g_addr_range(&b, &n, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
        return fail(MOK_ERR_INVALID, "cuMemGetAddressRange: not a device allocation");
    *base = reinterpret_cast<char *>(b);
    return MOK_OK;
}

int moe_ep_ipc_handle(const void *dev_ptr, void *handle, size_t *offset)
{
    if (!dev_ptr || !handle || !offset) return MOK_ERR_INVALID;
    static_assert(sizeof(cudaIpcMemHandle_t) == MOK_EP_IPC_HANDLE_BYTES, "IPC handle size");
    char *base = nullptr;
    MOK_TRY(ep_alloc_base(dev_ptr, &base));
    cudaIpcMemHandle_t h;
    if (const cudaError_t e = cudaIpcGetMemHandle(&h, base); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaIpcGetMemHandle", e);
    std::memcpy(handle, &h, sizeof(h));
    *offset = static_cast<size_t>(static_cast<const char *>(dev_ptr) - base);
    return MOK_OK;
}

int moe_ep_ipc_open(const void *handle, size_t offset, void **dev_ptr)
{
    if (!handle || !dev_ptr) return MOK_ERR_INVALID;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void *base = nullptr;
    if (const cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaIpcOpenMemHandle", e);
    *dev_ptr = static_cast<char *>(base) + offset;
    return MOK_OK;
}

int moe_ep_ipc_close(void *dev_ptr, size_t offset)
{
    if (!dev_ptr) return MOK_ERR_INVALID;
    if (const cudaError_t e = cudaIpcCloseMemHandle(static_cast<char *>(dev_ptr) - offset); e != cudaSuccess)
        return fail(MOK_ERR_LAUNCH, "cudaIpcCloseMemHandle", e);
    return MOK_OK;
}

int moe_set_schedule(int schedule)
{
    if (schedule != MOK_SCHEDULE_PERSISTENT && schedule != MOK_SCHEDULE_SPLIT && schedule != MOK_SCHEDULE_SPLIT_PDL)
        return MOK_ERR_INVALID;
    t_schedule = schedule;
    return MOK_OK;
}

int moe_get_schedule(int *schedule)
{
    if (!schedule) return MOK_ERR_INVALID;
    *schedule = t_schedule;
    return MOK_OK;
}

int moe_trace_device(void *buf, size_t bytes, void *bwd_buf, size_t bwd_bytes)
{
    if ((buf && !aligned16(buf)) || (bwd_buf && !aligned16(bwd_buf))) return MOK_ERR_INVALID;
    t_dev_trace = static_cast<unsigned long long *>(buf);
    t_dev_trace_bytes = buf ? bytes : 0;
    t_dev_trace_bwd = static_cast<unsigned long long *>(bwd_buf);
    t_dev_trace_bwd_bytes = bwd_buf ? bwd_bytes : 0;
    return MOK_OK;
}

int moe_launch_count(int *count)
{
    if (!count) return MOK_ERR_INVALID;
    *count = t_launches;
    return MOK_OK;
}

int moe_test_drop_signal(int enable)
{
    t_drop_signal = enable != 0;
    return MOK_OK;
}

const char *moe_last_error(void) { return t_last_error; }

const char *moe_strerror(int code)
{
    switch (code) {
    case MOK_OK: return "ok";
    case MOK_ERR_INVALID: return "invalid argument (shape, pointer, alignment or option)";
    case MOK_ERR_DEVICE: return "current device is not an sm_100 (B200) GPU";
    case MOK_ERR_WORKSPACE: return "ctx or scratch buffer too small";
    case MOK_ERR_LAUNCH: return "a CUDA call failed while enqueueing work";
    case MOK_ERR_UNSUPPORTED: return "combination not supported";
    default: return "unknown error";
    }
}

}  // extern "C"
