// libcpattn: the C ABI declared in include/cp_attn.h.  Host-side argument
// checks, workspace accounting, tensor-map encoding and kernel launches.  The
// library is one translation unit; the kernels live in the included headers.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "cp_attn.h"
#include "ptx.cuh"
#include "exp2_poly.cuh"
#include "tmap.h"
#include "zigzag.cuh"
#include "plan.cuh"
#include "merge.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "bwd_fused.cuh"
#include "fwd256.cuh"
#include "bwd256.cuh"

using namespace cpattn;

namespace {

constexpr int32_t kVersion = 100;  // 0.1.0

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device state.  Kernel attributes (the large dynamic shared-memory opt-in)
// and the SM count belong to a device, not to the process: a process that drives
// several GPUs sets them once on each, on first use with that device current.
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_num_sms[kMaxDevices] = {};
uint32_t g_attr_done[kMaxDevices] = {};   // bit per kernel family (AttrSet)

enum AttrSet : uint32_t {
    ATTR_FWD64 = 1, ATTR_FWD128 = 2, ATTR_BWD64 = 4, ATTR_BWD128 = 8, ATTR_FUSED64 = 16, ATTR_FUSED128 = 32,
    ATTR_FWD256 = 64, ATTR_BWD256 = 128, ATTR_MERGE_TILED = 256
};

inline int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

int num_sms()
{
    const int dev = current_device();
    if (dev < 0) return 148;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

// Run `set` (which applies cudaFuncSetAttribute to one kernel family) once per
// device; a failure is reported and retried on the next call.
template <typename F>
cp_status_t ensure_attr(AttrSet which, F set)
{
    const int dev = current_device();
    if (dev < 0) return CP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_attr_done[dev] & which) return CP_OK;
    if (set() != cudaSuccess) return CP_ERR_CUDA;
    g_attr_done[dev] |= which;
    return CP_OK;
}

// Checks shared by every call that takes a cp_problem_t.
cp_status_t check_problem(const cp_problem_t* p)
{
    if (!p) return CP_ERR_INVALID_ARG;
    if (p->batch < 1 || p->seq_len < 1 || p->cp_size < 1 || p->num_heads < 1 ||
        p->num_kv_heads < 1 || p->head_dim < 1)
        return CP_ERR_INVALID_ARG;
    if (p->seq_len % (2 * p->cp_size) != 0) return CP_ERR_INVALID_ARG;
    if (p->num_heads % p->num_kv_heads != 0) return CP_ERR_INVALID_ARG;
    if (p->rotate != CP_ROTATE_ALLGATHER && p->rotate != CP_ROTATE_RING) return CP_ERR_INVALID_ARG;
    if (p->mask != CP_MASK_CAUSAL && p->mask != CP_MASK_DOC_CAUSAL && p->mask != CP_MASK_FULL)
        return CP_ERR_INVALID_ARG;
    if (p->merge != CP_MERGE_SEPARATE && p->merge != CP_MERGE_FUSED) return CP_ERR_INVALID_ARG;
    if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale)) return CP_ERR_INVALID_ARG;
    if (p->window < 0) return CP_ERR_INVALID_ARG;
    // without the causal mask: no documents, and a window (one-sided) is not defined
    if (p->mask == CP_MASK_FULL && (p->cu_seqlens || p->num_docs != 0)) return CP_ERR_INVALID_ARG;
    if (p->mask == CP_MASK_FULL && p->window != 0) return CP_ERR_UNSUPPORTED;
    if (p->shard != CP_SHARD_SEQUENCE && p->shard != CP_SHARD_PER_DOC) return CP_ERR_INVALID_ARG;
    if (p->shard == CP_SHARD_PER_DOC && p->mask != CP_MASK_DOC_CAUSAL) return CP_ERR_INVALID_ARG;
    if (p->mask == CP_MASK_DOC_CAUSAL) {
        if (!p->cu_seqlens || p->num_docs < 1 || p->num_docs > p->seq_len) return CP_ERR_INVALID_ARG;
    }
    if (p->cp_size > PLAN_MAX_CP) return CP_ERR_UNSUPPORTED;
    // every flat row index (batch*heads*seq) and element offset must fit the kernels' types
    const int64_t rows = static_cast<int64_t>(p->batch) * p->num_heads * p->seq_len;
    if (rows > (int64_t(1) << 31) - 1) return CP_ERR_UNSUPPORTED;
    return CP_OK;
}

cp_status_t check_attention(const cp_problem_t* p)
{
    cp_status_t st = check_problem(p);
    if (st != CP_OK) return st;
    if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return CP_ERR_UNSUPPORTED;
    // the kernels' tile bounds (key tile end + window or sequence length) stay in int32
    if (p->seq_len > (1 << 29)) return CP_ERR_UNSUPPORTED;
    const int C = p->seq_len / (2 * p->cp_size);
    if (C % 128 != 0) return CP_ERR_UNSUPPORTED;
    return CP_OK;
}

cp_status_t check_plan(const cp_plan_t* pl, bool need_all, const cp_problem_t* p = nullptr)
{
    if (!pl) return CP_ERR_INVALID_ARG;
    if (!pl->src || !pl->doc_start) return CP_ERR_INVALID_ARG;
    if (need_all && (!pl->perm || !pl->inv_perm || !pl->rank_cu_off || !pl->rank_cu || !pl->pairs ||
                     !pl->tile_orig || !pl->tile_shard))
        return CP_ERR_INVALID_ARG;
    // per-document plans: the attention kernels read the tile tables
    if (p && p->shard == CP_SHARD_PER_DOC && (!pl->tile_orig || !pl->tile_shard)) return CP_ERR_INVALID_ARG;
    return CP_OK;
}

// The tile tables for the attention kernels: only per-document plans need them.
inline const int32_t* tables_orig(const cp_problem_t* p, const cp_plan_t* pl)
{
    return p->shard == CP_SHARD_PER_DOC ? pl->tile_orig : nullptr;
}
inline const int32_t* tables_shard(const cp_problem_t* p, const cp_plan_t* pl)
{
    return p->shard == CP_SHARD_PER_DOC ? pl->tile_shard : nullptr;
}

// Keys visible to the query at original position q start at q - wm1 (window W:
// wm1 = W - 1); without a window wm1 is larger than any position, so the bound
// never binds.
inline int32_t window_minus_one(const cp_problem_t* p)
{
    return p->window > 0 ? p->window - 1 : p->seq_len + 256;
}

// Last visible key of the query at original position q is q + nc: nc = 0 under
// the causal mask; nc = S (beyond every key) without it.
inline int32_t noncausal_shift(const cp_problem_t* p)
{
    return p->mask == CP_MASK_FULL ? p->seq_len : 0;
}

inline float softmax_scale(const cp_problem_t* p)
{
    return p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace handshake shared by every call that takes (ws, ws_bytes).
// Returns true when the caller should return `out` right away.
inline bool workspace_gate(size_t need, void* ws, size_t* ws_bytes, cp_status_t* out)
{
    if (ws_bytes && !ws) { *ws_bytes = need; *out = CP_OK; return true; }
    if (need == 0) return false;
    if (!ws || !ws_bytes) { *out = CP_ERR_INVALID_ARG; return true; }
    if (*ws_bytes < need) { *out = CP_ERR_WORKSPACE; return true; }
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) { *out = CP_ERR_INVALID_ARG; return true; }
    return false;
}

inline cp_status_t launch_status()
{
    return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

// ---- launch counter and optional event trace (see cp_trace_begin)
int64_t g_launches = 0;
cudaEvent_t* g_trace_events = nullptr;
int32_t g_trace_cap = 0, g_trace_n = 0;
int32_t g_trace_ids[4096];
constexpr int32_t kTraceMax = 4096;

struct LaunchScope {
    cudaStream_t s;
    bool traced;
    LaunchScope(int kernel, cudaStream_t stream) : s(stream), traced(false)
    {
        ++g_launches;
        if (g_trace_events) {
            if (g_trace_n < g_trace_cap) {
                cudaEventRecord(g_trace_events[2 * g_trace_n], s);
                traced = true;
            }
            if (g_trace_n < kTraceMax) g_trace_ids[g_trace_n] = kernel;
        }
    }
    ~LaunchScope()
    {
        if (traced) cudaEventRecord(g_trace_events[2 * g_trace_n + 1], s);
        if (g_trace_events) ++g_trace_n;
    }
};

cp_status_t launch_gather(const cp_problem_t* p, const cp_plan_t* pl, int32_t n_bufs,
                          const void* const* bufs_in, void* const* bufs_out,
                          const int64_t* buf_outer, const int64_t* buf_row_bytes, int to_shard,
                          cudaStream_t stream)
{
    const int C = p->seq_len / (2 * p->cp_size);
    for (int i = 0; i < n_bufs; ++i) {
        if (buf_outer[i] == 0) continue;
        GatherParams G;
        G.in = static_cast<const uint4*>(bufs_in[i]);
        G.out = static_cast<uint4*>(bufs_out[i]);
        G.rows = buf_outer[i] * p->seq_len;
        G.vpr = static_cast<int32_t>(buf_row_bytes[i] / 16);
        G.rpw = (G.vpr <= 32 && 32 % G.vpr == 0) ? 32 / G.vpr : 1;
        G.S = p->seq_len;
        G.C = C;
        G.cp = p->cp_size;
        G.to_shard = to_shard;
        // per-document shards have no closed form: the plan's permutation tables
        G.map = p->shard == CP_SHARD_PER_DOC ? (to_shard ? pl->perm : pl->inv_perm) : nullptr;
        const int64_t warps_needed = (G.rows + G.rpw * 4 - 1) / (G.rpw * 4);
        const int64_t blocks = std::min<int64_t>((warps_needed + 7) / 8, int64_t(num_sms()) * 8);
        LaunchScope ls(CP_K_GATHER, stream);
        const unsigned grid = static_cast<unsigned>(std::max<int64_t>(blocks, 1));
        if (G.map)
            gather_rows_kernel<true><<<grid, 256, 0, stream>>>(G);
        else
            gather_rows_kernel<false><<<grid, 256, 0, stream>>>(G);
        if (launch_status() != CP_OK) return CP_ERR_CUDA;
    }
    return CP_OK;
}

cp_status_t check_bufs(const cp_problem_t* p, int32_t n_bufs, const void* const* bufs_in,
                       void* const* bufs_out, const int64_t* buf_outer,
                       const int64_t* buf_row_bytes)
{
    if (n_bufs < 0 || n_bufs > 16) return CP_ERR_INVALID_ARG;
    if (n_bufs == 0) return CP_OK;
    if (!bufs_in || !bufs_out || !buf_outer || !buf_row_bytes) return CP_ERR_INVALID_ARG;
    for (int i = 0; i < n_bufs; ++i) {
        if (buf_outer[i] < 0 || buf_row_bytes[i] <= 0 || buf_row_bytes[i] % 16 != 0)
            return CP_ERR_INVALID_ARG;
        if (buf_outer[i] == 0) continue;
        if (!bufs_in[i] || !bufs_out[i] || !aligned16(bufs_in[i]) || !aligned16(bufs_out[i]))
            return CP_ERR_INVALID_ARG;
        if (buf_outer[i] * static_cast<int64_t>(p->seq_len) > (int64_t(1) << 40))
            return CP_ERR_UNSUPPORTED;
        const uintptr_t a = reinterpret_cast<uintptr_t>(bufs_in[i]);
        const uintptr_t b = reinterpret_cast<uintptr_t>(bufs_out[i]);
        const uintptr_t n = static_cast<uintptr_t>(buf_outer[i] * p->seq_len * buf_row_bytes[i]);
        if (a < b + n && b < a + n) return CP_ERR_INVALID_ARG;  // in/out overlap
    }
    return CP_OK;
}

// Which rows a launch covers and how its tensors are laid out: the whole
// sequence (every rank, every step, tensors of S rows per head), or one rank's
// local query shard (2C rows per head, first row at shard position r*2C) against
// gathered K/V (S rows) or against the single K/V shard of one ring step (2C rows).
struct Layout {
    int32_t q_rows, q_base, kv_rows, kv_base, rank, s0, s1;
};

inline Layout whole_layout(const cp_problem_t* p)
{
    return Layout{p->seq_len, 0, p->seq_len, 0, -1, 0, p->cp_size};
}

inline Layout rank_layout(const cp_problem_t* p, int rank, int step)
{
    const int n2c = p->seq_len / p->cp_size;
    if (step < 0) return Layout{n2c, rank * n2c, p->seq_len, 0, rank, 0, p->cp_size};
    return Layout{n2c, rank * n2c, n2c, -1, rank, step, step + 1};
}

template <int D>
cp_status_t launch_fwd(const cp_problem_t* p, const cp_plan_t* pl, const void* q, const void* k,
                       const void* v, void* o, float* lse, float* o_parts, float* lse_parts,
                       cudaStream_t stream, int stall, const Layout& L, bool fused)
{
    const int B = p->batch, Hq = p->num_heads, Hkv = p->num_kv_heads, S = p->seq_len;
    // head_dim 256: 64-row K/V boxes, Q read by the kernel itself (into tensor memory)
    constexpr int KV_BOX_ROWS = D == 256 ? Fwd256Cfg::KT : 128;
    CUtensorMap tq, tk, tv;
    if ((D != 256 && !make_tmap_bf16_2d(&tq, q, D, static_cast<uint64_t>(B) * Hq * L.q_rows, D * 2, 64, 128)) ||
        !make_tmap_bf16_2d(&tk, k, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, KV_BOX_ROWS) ||
        !make_tmap_bf16_2d(&tv, v, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, KV_BOX_ROWS))
        return CP_ERR_CUDA;
    FwdParams P;
    P.BH = B * Hq;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.S = S;
    P.cp = p->cp_size;
    P.C = S / (2 * p->cp_size);
    P.docs = p->mask == CP_MASK_DOC_CAUSAL;
    P.wm1 = window_minus_one(p);
    P.nc = noncausal_shift(p);
    P.fused = fused;
    P.scale_log2 = softmax_scale(p) * 1.4426950408889634f;
    P.ppc = (P.C + 255) / 256;
    // per-document shards: work units of 256 shard rows (two 128-row query
    // tiles, not necessarily adjacent in the original order)
    P.n_items = p->shard == CP_SHARD_PER_DOC ? P.BH * (L.q_rows / 256)
                                              : P.BH * (L.rank < 0 ? 2 * P.cp : 2) * P.ppc;
    P.tile_orig = tables_orig(p, pl);
    P.tile_shard = tables_shard(p, pl);
    P.stall = stall;
    P.q_rows = L.q_rows;
    P.q_base = L.q_base;
    P.kv_rows = L.kv_rows;
    P.kv_base = L.kv_base;
    P.rank = L.rank;
    P.s0 = L.s0;
    P.s1 = L.s1;
    P.src = pl->src;
    P.doc_start = pl->doc_start;
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.o = static_cast<__nv_bfloat16*>(o);
    P.lse = lse;
    P.o_parts = o_parts;
    P.lse_parts = lse_parts;
    // partials into the caller's buffers (cp_attn_fwd_step: no o) stay row-major;
    // the library's own workspace is tile-interleaved for lse_merge_tiled_kernel
    P.parts_tiled = o != nullptr;
    if constexpr (D == 256) {
        // one 128-row query tile per work item
        P.n_items = P.BH * (L.q_rows / 128);
        const cp_status_t ast = ensure_attr(ATTR_FWD256, [] {
            cudaError_t e = cudaFuncSetAttribute(cp_fwd256_kernel<false>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 Fwd256Cfg::SMEM_BYTES);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(cp_fwd256_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Fwd256Cfg::SMEM_BYTES);
            return e;
        });
        if (ast != CP_OK) return ast;
        const int grid = std::min(P.n_items, num_sms());
        LaunchScope ls(CP_K_FWD, stream);
        auto* kern = p->shard == CP_SHARD_PER_DOC ? cp_fwd256_kernel<true> : cp_fwd256_kernel<false>;
        kern<<<grid, Fwd256Cfg::THREADS, Fwd256Cfg::SMEM_BYTES, stream>>>(tk, tv, P);
        return launch_status();
    } else {
    using Cfg = FwdCfg<D>;
    const cp_status_t ast = ensure_attr(D == 128 ? ATTR_FWD128 : ATTR_FWD64, [] {
        cudaError_t e = cudaFuncSetAttribute(cp_fwd_kernel<D, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(cp_fwd_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM_BYTES);
        return e;
    });
    if (ast != CP_OK) return ast;
    const int grid = std::min(P.n_items, num_sms());
    LaunchScope ls(CP_K_FWD, stream);
    // per-document plans take the instantiation that reads the tile tables
    auto* kern = p->shard == CP_SHARD_PER_DOC ? cp_fwd_kernel<D, true> : cp_fwd_kernel<D, false>;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tq, tk, tv, P);
    return launch_status();
    }
}

// The forward for the problem's head_dim.
cp_status_t launch_fwd_any(const cp_problem_t* p, const cp_plan_t* pl, const void* q, const void* k,
                           const void* v, void* o, float* lse, float* o_parts, float* lse_parts,
                           cudaStream_t stream, int stall, const Layout& L, bool fused)
{
    switch (p->head_dim) {
    case 256: return launch_fwd<256>(p, pl, q, k, v, o, lse, o_parts, lse_parts, stream, stall, L, fused);
    case 128: return launch_fwd<128>(p, pl, q, k, v, o, lse, o_parts, lse_parts, stream, stall, L, fused);
    default: return launch_fwd<64>(p, pl, q, k, v, o, lse, o_parts, lse_parts, stream, stall, L, fused);
    }
}

cp_status_t launch_merge(int64_t rows, int32_t D, int32_t n_parts, const float* o_parts,
                         const float* lse_parts, void* o_out, float* lse_out, cudaStream_t stream,
                         bool tiled = false)
{
    if (rows == 0) return CP_OK;
    MergeParams M;
    M.rows = rows;
    M.D = D;
    M.n_parts = n_parts;
    M.o_parts = o_parts;
    M.lse_parts = lse_parts;
    M.o_out = static_cast<__nv_bfloat16*>(o_out);
    M.lse_out = lse_out;
    if (tiled) {
        // the forward's own partials (rows a multiple of 128, tile-interleaved)
        const cp_status_t ast = ensure_attr(ATTR_MERGE_TILED, [] {
            return cudaFuncSetAttribute(lse_merge_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        232448);
        });
        if (ast != CP_OK) return ast;
        const size_t smem = size_t(n_parts) * 128 * 4 + 128 * 4 + size_t(128) * (D / 4 + 1) * 8;
        const int64_t blocks = std::min<int64_t>(rows / 128, int64_t(num_sms()) * 8);
        LaunchScope ls(CP_K_MERGE, stream);
        lse_merge_tiled_kernel<<<static_cast<unsigned>(blocks), 256, smem, stream>>>(M);
        return launch_status();
    }
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, int64_t(num_sms()) * 16);
    LaunchScope ls(CP_K_MERGE, stream);
    lse_merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(M);
    return launch_status();
}

__global__ void selftest_wait_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
        // nothing ever arrives on this barrier: the bounded wait must give up
        mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, limit_ns);
    }
}

__global__ void selftest_exp2_kernel(const float* x, float* ys, float* yh, int64_t n)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        ys[i] = exp2_poly(x[i]);
        yh[i] = ex2_approx(x[i]);
    }
}

}  // namespace

extern "C" {

int32_t cp_version(void) { return kVersion; }

cp_status_t cp_selftest_exp2(const float* x, float* y_soft, float* y_hw, int64_t n, void* stream)
{
    if (n < 0) return CP_ERR_INVALID_ARG;
    if (n == 0) return CP_OK;
    if (!x || !y_soft || !y_hw) return CP_ERR_INVALID_ARG;
    LaunchScope ls(CP_K_SELFTEST_EXP2, as_stream(stream));
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, int64_t(num_sms()) * 8);
    selftest_exp2_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(x, y_soft, y_hw, n);
    return launch_status();
}

int64_t cp_launch_count(void) { return g_launches; }

cp_status_t cp_trace_begin(void* const* events, int32_t capacity)
{
    if (!events || capacity < 1) return CP_ERR_INVALID_ARG;
    for (int32_t i = 0; i < 2 * capacity; ++i)
        if (!events[i]) return CP_ERR_INVALID_ARG;
    g_trace_events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
    g_trace_cap = capacity;
    g_trace_n = 0;
    return CP_OK;
}

cp_status_t cp_trace_end(int32_t* n_launches, int32_t* kernel_ids)
{
    if (!n_launches) return CP_ERR_INVALID_ARG;
    *n_launches = g_trace_n;
    if (kernel_ids)
        for (int32_t i = 0; i < std::min(g_trace_n, std::min(g_trace_cap, kTraceMax)); ++i)
            kernel_ids[i] = g_trace_ids[i];
    g_trace_events = nullptr;
    g_trace_cap = 0;
    g_trace_n = 0;
    return CP_OK;
}

cp_status_t cp_plan_shards(const cp_problem_t* problem, const cp_plan_t* plan, int32_t n_bufs,
                           const void* const* bufs_in, void* const* bufs_out,
                           const int64_t* buf_outer, const int64_t* buf_row_bytes, void* ws,
                           size_t* ws_bytes, void* stream)
{
    cp_status_t st = check_problem(problem);
    if (st != CP_OK) return st;
    if ((st = check_plan(plan, true)) != CP_OK) return st;
    if ((st = check_bufs(problem, n_bufs, bufs_in, bufs_out, buf_outer, buf_row_bytes)) != CP_OK)
        return st;
    if (workspace_gate(0, ws, ws_bytes, &st)) return st;
    cudaStream_t s = as_stream(stream);
    PlanParams P;
    P.S = problem->seq_len;
    P.cp = problem->cp_size;
    P.C = P.S / (2 * P.cp);
    P.docs = problem->mask == CP_MASK_DOC_CAUSAL;
    P.wm1 = window_minus_one(problem);
    P.causal = problem->mask != CP_MASK_FULL;
    P.num_docs = P.docs ? problem->num_docs : 1;
    P.rotate = problem->rotate;
    P.cu = problem->cu_seqlens;
    P.perm = plan->perm;
    P.inv_perm = plan->inv_perm;
    P.src = plan->src;
    P.doc_start = plan->doc_start;
    P.rank_cu_off = plan->rank_cu_off;
    P.rank_cu = plan->rank_cu;
    P.pairs = plan->pairs;
    P.per_doc = problem->shard == CP_SHARD_PER_DOC;
    P.tile_orig = plan->tile_orig;
    P.tile_shard = plan->tile_shard;
    {
        LaunchScope ls(CP_K_PLAN_META, s);
        plan_meta_kernel<<<1, 256, 0, s>>>(P);
    }
    if (launch_status() != CP_OK) return CP_ERR_CUDA;
    const int blocks = std::min((P.S + 255) / 256, num_sms() * 8);
    {
        LaunchScope ls(CP_K_PLAN_INDEX, s);
        plan_index_kernel<<<blocks, 256, 0, s>>>(P);
    }
    if (launch_status() != CP_OK) return CP_ERR_CUDA;
    return launch_gather(problem, plan, n_bufs, bufs_in, bufs_out, buf_outer, buf_row_bytes, 1, s);
}

cp_status_t cp_unshard(const cp_problem_t* problem, const cp_plan_t* plan, int32_t n_bufs,
                       const void* const* bufs_in, void* const* bufs_out,
                       const int64_t* buf_outer, const int64_t* buf_row_bytes, void* stream)
{
    cp_status_t st = check_problem(problem);
    if (st != CP_OK) return st;
    if (!plan) return CP_ERR_INVALID_ARG;
    if (problem->shard == CP_SHARD_PER_DOC && !plan->inv_perm) return CP_ERR_INVALID_ARG;
    if ((st = check_bufs(problem, n_bufs, bufs_in, bufs_out, buf_outer, buf_row_bytes)) != CP_OK)
        return st;
    return launch_gather(problem, plan, n_bufs, bufs_in, bufs_out, buf_outer, buf_row_bytes, 0,
                         as_stream(stream));
}

}  // extern "C"

namespace {

cp_status_t attn_fwd_impl(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                          const void* k, const void* v, void* o, float* lse, void* ws,
                          size_t* ws_bytes, void* stream, int stall)
{
    cp_status_t st = check_attention(problem);
    if (st != CP_OK) return st;
    if ((st = check_plan(plan, false, problem)) != CP_OK) return st;
    if (!q || !k || !v || !o || !lse) return CP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return CP_ERR_INVALID_ARG;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * problem->seq_len;
    const bool separate = problem->merge == CP_MERGE_SEPARATE;
    const size_t o_parts_bytes = separate ? round_up(size_t(problem->cp_size) * rows * problem->head_dim * 4, 256) : 0;
    const size_t lse_parts_bytes = separate ? round_up(size_t(problem->cp_size) * rows * 4, 256) : 0;
    if (workspace_gate(o_parts_bytes + lse_parts_bytes, ws, ws_bytes, &st)) return st;
    float* o_parts = separate ? static_cast<float*>(ws) : nullptr;
    float* lse_parts = separate ? reinterpret_cast<float*>(static_cast<char*>(ws) + o_parts_bytes) : nullptr;
    cudaStream_t s = as_stream(stream);
    const Layout L = whole_layout(problem);
    const bool fused = problem->merge == CP_MERGE_FUSED;
    st = launch_fwd_any(problem, plan, q, k, v, o, lse, o_parts, lse_parts, s, stall, L, fused);
    if (st != CP_OK || !separate) return st;
    return launch_merge(rows, problem->head_dim, problem->cp_size, o_parts, lse_parts, o, lse, s, true);
}

}  // namespace

extern "C" {

cp_status_t cp_attn_fwd(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                        const void* k, const void* v, void* o, float* lse, void* ws,
                        size_t* ws_bytes, void* stream)
{
    return attn_fwd_impl(problem, plan, q, k, v, o, lse, ws, ws_bytes, stream, 0);
}

cp_status_t cp_lse_merge(int64_t rows, int32_t head_dim, int32_t n_parts, const float* o_parts,
                         const float* lse_parts, void* o_out, float* lse_out, void* stream)
{
    if (rows < 0 || head_dim < 4 || head_dim > 256 || head_dim % 4 != 0) return CP_ERR_INVALID_ARG;
    if (n_parts < 1 || n_parts > MERGE_MAX_PARTS) return CP_ERR_INVALID_ARG;
    if (rows == 0) return CP_OK;
    if (!o_parts || !lse_parts || !o_out || !lse_out) return CP_ERR_INVALID_ARG;
    if (!aligned16(o_parts) || !aligned16(o_out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
        (reinterpret_cast<uintptr_t>(lse_out) & 3u))
        return CP_ERR_INVALID_ARG;
    return launch_merge(rows, head_dim, n_parts, o_parts, lse_parts, o_out, lse_out, as_stream(stream));
}

cp_status_t cp_get_device_status(int32_t* status, void* stream)
{
    if (!status) return CP_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    int32_t v = 0;
    const int32_t zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_cp_device_status, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return CP_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CP_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(g_cp_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return CP_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CP_ERR_CUDA;
    *status = v;
    return CP_OK;
}

cp_status_t cp_set_wait_limit_ns(uint64_t limit_ns)
{
    if (limit_ns == 0) return CP_ERR_INVALID_ARG;
    const unsigned long long v = limit_ns;
    if (cudaMemcpyToSymbol(g_cp_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return CP_ERR_CUDA;
    return CP_OK;
}

cp_status_t cp_selftest_wait_timeout(uint64_t limit_ns, void* stream)
{
    if (limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000) return CP_ERR_INVALID_ARG;
    LaunchScope ls(CP_K_SELFTEST, as_stream(stream));
    selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns);
    return launch_status();
}

}  // extern "C"

namespace {

template <int D>
cp_status_t launch_bwd(const cp_problem_t* p, const cp_plan_t* pl, const void* q, const void* k,
                       const void* v, const void* o, const float* lse, const void* dout, void* dq,
                       void* dk, void* dv, float* delta, float* nlse2, cudaStream_t stream,
                       int stall, const Layout& L, float* dk32, float* dv32, float* dq_acc,
                       float* dq32 = nullptr, bool ring_step = false)
{
    // dq_acc non-null: the one-pass backward (cp_bwd_fused_kernel + dq_convert_kernel);
    // null: the two deterministic passes (cp_bwd_dkdv_kernel, cp_bwd_dq_kernel)
    const int B = p->batch, Hq = p->num_heads, Hkv = p->num_kv_heads, S = p->seq_len;
    const int64_t rows = static_cast<int64_t>(B) * Hq * L.q_rows;
    {
        const int64_t blocks = std::min<int64_t>((rows + 7) / 8, int64_t(num_sms()) * 16);
        LaunchScope ls(CP_K_BWD_PREP, stream);
        bwd_prep_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, delta,
            nlse2, rows, D, dq_acc);
        if (launch_status() != CP_OK) return CP_ERR_CUDA;
    }
    // head_dim 256: the dK / dV passes stream 64-row query units
    constexpr int QBOX_ROWS = D == 256 ? Kv256Cfg<0>::QT : 128;
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tmap_bf16_2d(&tq, q, D, static_cast<uint64_t>(B) * Hq * L.q_rows, D * 2, 64, QBOX_ROWS) ||
        !make_tmap_bf16_2d(&tk, k, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, 128) ||
        !make_tmap_bf16_2d(&tv, v, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, 128) ||
        !make_tmap_bf16_2d(&tdo, dout, D, static_cast<uint64_t>(B) * Hq * L.q_rows, D * 2, 64, QBOX_ROWS))
        return CP_ERR_CUDA;
    BwdParams P;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.S = S;
    P.cp = p->cp_size;
    P.C = S / (2 * p->cp_size);
    P.docs = p->mask == CP_MASK_DOC_CAUSAL;
    P.wm1 = window_minus_one(p);
    P.nc = noncausal_shift(p);
    P.scale = softmax_scale(p);
    P.scale_log2 = P.scale * 1.4426950408889634f;
    P.src = pl->src;
    P.doc_start = pl->doc_start;
    P.cu = p->cu_seqlens;
    P.num_docs = P.docs ? p->num_docs : 0;
    P.nlse2 = nlse2;
    P.delta = delta;
    P.q = static_cast<const __nv_bfloat16*>(q);
    P.dout = static_cast<const __nv_bfloat16*>(dout);
    P.dq = static_cast<__nv_bfloat16*>(dq);
    P.dk = static_cast<__nv_bfloat16*>(dk);
    P.dv = static_cast<__nv_bfloat16*>(dv);
    P.stall = stall;
    P.q_rows = L.q_rows;
    P.q_base = L.q_base;
    P.kv_rows = L.kv_rows;
    P.kv_base = L.kv_base;
    P.rank = L.rank;
    P.dk32 = dk32;
    P.dv32 = dv32;
    P.dq_acc = dq_acc;
    P.s0 = L.s0;
    P.s1 = L.s1;
    // one ring step: the dK/dV pass covers the shard visited at that step, and dQ, dK,
    // dV are added into the caller's fp32 sums
    P.step_shard = ring_step;
    P.accumulate = ring_step;
    P.dq32 = dq32;
    P.tile_orig = tables_orig(p, pl);
    P.tile_shard = tables_shard(p, pl);
    const bool pd = p->shard == CP_SHARD_PER_DOC;
    if constexpr (D == 256) {
        // three passes: dV, dK (64-row query units against 128-key tiles), dQ (64-key
        // tiles against 128-row query tiles); no one-pass form
        if (dq_acc) return CP_ERR_UNSUPPORTED;
        CUtensorMap tk64, tv64, tdo128;
        if (!make_tmap_bf16_2d(&tk64, k, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, Dq256Cfg::KT) ||
            !make_tmap_bf16_2d(&tv64, v, D, static_cast<uint64_t>(B) * Hkv * L.kv_rows, D * 2, 64, Dq256Cfg::KT) ||
            !make_tmap_bf16_2d(&tdo128, dout, D, static_cast<uint64_t>(B) * Hq * L.q_rows, D * 2, 64, 128))
            return CP_ERR_CUDA;
        const cp_status_t ast = ensure_attr(ATTR_BWD256, [] {
            cudaError_t e = cudaSuccess;
            for (auto* kd : {cp_bwd256_kv_kernel<false, 0>, cp_bwd256_kv_kernel<true, 0>})
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, Kv256Cfg<0>::SMEM_BYTES);
            for (auto* kd : {cp_bwd256_kv_kernel<false, 1>, cp_bwd256_kv_kernel<true, 1>})
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, Kv256Cfg<1>::SMEM_BYTES);
            for (auto* kq : {cp_bwd256_dq_kernel<false>, cp_bwd256_dq_kernel<true>})
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, Dq256Cfg::SMEM_BYTES);
            return e;
        });
        if (ast != CP_OK) return ast;
        P.n_items = B * Hkv * (ring_step ? P.C / 128 : S / 256);   // pairs of key tiles
        const int grid_kv = std::min(P.n_items, num_sms());
        {
            LaunchScope ls(CP_K_BWD_DKDV, stream);
            auto* kv = pd ? cp_bwd256_kv_kernel<true, 0> : cp_bwd256_kv_kernel<false, 0>;
            kv<<<grid_kv, BWD_THREADS, Kv256Cfg<0>::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, P);
        }
        if (launch_status() != CP_OK) return CP_ERR_CUDA;
        {
            LaunchScope ls(CP_K_BWD_DKDV, stream);
            auto* kk = pd ? cp_bwd256_kv_kernel<true, 1> : cp_bwd256_kv_kernel<false, 1>;
            kk<<<grid_kv, BWD_THREADS, Kv256Cfg<1>::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, P);
        }
        if (launch_status() != CP_OK) return CP_ERR_CUDA;
        P.n_items = B * Hq * (L.q_rows / 128);
        LaunchScope ls(CP_K_BWD_DQ, stream);
        auto* kq = pd ? cp_bwd256_dq_kernel<true> : cp_bwd256_dq_kernel<false>;
        kq<<<std::min(P.n_items, num_sms()), BWD_THREADS, Dq256Cfg::SMEM_BYTES, stream>>>(tk64, tv64, tdo128, P);
        return launch_status();
    } else {
    const cp_status_t ast = ensure_attr(D == 128 ? ATTR_BWD128 : ATTR_BWD64, [] {
        cudaError_t e = cudaSuccess;
        for (auto* kd : {cp_bwd_dkdv_kernel<D, false>, cp_bwd_dkdv_kernel<D, true>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, DkdvCfg<D>::SMEM_BYTES);
        for (auto* kq : {cp_bwd_dq_kernel<D, false>, cp_bwd_dq_kernel<D, true>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, DqCfg<D>::SMEM_BYTES);
        return e;
    });
    if (ast != CP_OK) return ast;
    P.n_items = B * Hkv * (ring_step ? P.C / 128 : S / 256);   // pairs of key tiles (S / 128 is even)
    if (dq_acc) {
        const cp_status_t fst = ensure_attr(D == 128 ? ATTR_FUSED128 : ATTR_FUSED64, [] {
            cudaError_t e = cudaFuncSetAttribute(cp_bwd_fused_kernel<D, false>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 FusedCfg<D>::SMEM_BYTES);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(cp_bwd_fused_kernel<D, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, FusedCfg<D>::SMEM_BYTES);
            return e;
        });
        if (fst != CP_OK) return fst;
        {
            LaunchScope ls(CP_K_BWD_FUSED, stream);
            auto* kern = pd ? cp_bwd_fused_kernel<D, true> : cp_bwd_fused_kernel<D, false>;
            kern<<<std::min(P.n_items, num_sms()), FusedCfg<D>::THREADS, FusedCfg<D>::SMEM_BYTES, stream>>>(
                tq, tk, tv, tdo, P);
        }
        if (launch_status() != CP_OK) return CP_ERR_CUDA;
        const int64_t n8 = rows * D / 8;
        const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, int64_t(num_sms()) * 8);
        LaunchScope ls(CP_K_DQ_CONVERT, stream);
        dq_convert_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            reinterpret_cast<const float4*>(dq_acc), static_cast<uint4*>(dq), n8, P.scale);
        return launch_status();
    }
    {
    LaunchScope ls(CP_K_BWD_DKDV, stream);
    auto* kdkdv = pd ? cp_bwd_dkdv_kernel<D, true> : cp_bwd_dkdv_kernel<D, false>;
    kdkdv<<<std::min(P.n_items, num_sms()), DkdvCfg<D>::THREADS, DkdvCfg<D>::SMEM_BYTES, stream>>>(
        tq, tk, tv, tdo, P);
    }
    if (launch_status() != CP_OK) return CP_ERR_CUDA;
    P.n_items = B * Hq * (L.q_rows / 128);
    LaunchScope ls(CP_K_BWD_DQ, stream);
    auto* kdq = pd ? cp_bwd_dq_kernel<D, true> : cp_bwd_dq_kernel<D, false>;
    kdq<<<std::min(P.n_items, num_sms()), DqCfg<D>::THREADS, DqCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, P);
    return launch_status();
    }
}

// The backward for the problem's head_dim.
cp_status_t launch_bwd_any(const cp_problem_t* p, const cp_plan_t* pl, const void* q, const void* k,
                           const void* v, const void* o, const float* lse, const void* dout, void* dq,
                           void* dk, void* dv, float* delta, float* nlse2, cudaStream_t stream,
                           int stall, const Layout& L, float* dk32, float* dv32, float* dq_acc,
                           float* dq32 = nullptr, bool ring_step = false)
{
    switch (p->head_dim) {
    case 256:
        return launch_bwd<256>(p, pl, q, k, v, o, lse, dout, dq, dk, dv, delta, nlse2, stream, stall, L,
                               dk32, dv32, dq_acc, dq32, ring_step);
    case 128:
        return launch_bwd<128>(p, pl, q, k, v, o, lse, dout, dq, dk, dv, delta, nlse2, stream, stall, L,
                               dk32, dv32, dq_acc, dq32, ring_step);
    default:
        return launch_bwd<64>(p, pl, q, k, v, o, lse, dout, dq, dk, dv, delta, nlse2, stream, stall, L,
                              dk32, dv32, dq_acc, dq32, ring_step);
    }
}

}  // namespace

namespace {

cp_status_t attn_bwd_impl(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                          const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, void* ws,
                          size_t* ws_bytes, void* stream, int stall)
{
    cp_status_t st = check_attention(problem);
    if (st != CP_OK) return st;
    if ((st = check_plan(plan, false, problem)) != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * problem->seq_len;
    const size_t row_bytes = round_up(size_t(rows) * 4, 256);
    // the two deterministic passes unless the caller asks for the one-pass form (the
    // stall hook picks the form of the kernel it targets)
    const bool one_pass = stall == CP_K_BWD_FUSED || (problem->bwd_one_pass && stall == 0);
    if (one_pass && problem->head_dim == 256) return CP_ERR_UNSUPPORTED;   // three passes only
    const size_t acc_bytes = one_pass ? round_up(size_t(rows) * problem->head_dim * 4, 256) : 0;
    if (workspace_gate(2 * row_bytes + acc_bytes, ws, ws_bytes, &st)) return st;
    float* delta = static_cast<float*>(ws);
    float* nlse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + row_bytes);
    float* dq_acc = one_pass ? reinterpret_cast<float*>(static_cast<char*>(ws) + 2 * row_bytes) : nullptr;
    cudaStream_t s = as_stream(stream);
    return launch_bwd_any(problem, plan, q, k, v, o, lse, dout, dq, dk, dv, delta, nlse2, s, stall, whole_layout(problem), nullptr, nullptr, dq_acc);
}

}  // namespace

extern "C" cp_status_t cp_attn_bwd(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                                   const void* k, const void* v, const void* o, const float* lse,
                                   const void* dout, void* dq, void* dk, void* dv, void* ws,
                                   size_t* ws_bytes, void* stream)
{
    return attn_bwd_impl(problem, plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, stream, 0);
}

extern "C" cp_status_t cp_selftest_stall(int32_t kernel, const cp_problem_t* problem,
                                         const cp_plan_t* plan, const void* q, const void* k,
                                         const void* v, void* o, float* lse, const void* dout,
                                         void* dq, void* dk, void* dv, void* ws, size_t* ws_bytes,
                                         void* stream)
{
    if (kernel == CP_K_FWD)
        return attn_fwd_impl(problem, plan, q, k, v, o, lse, ws, ws_bytes, stream, 1);
    if (kernel == CP_K_BWD_DKDV || kernel == CP_K_BWD_DQ || kernel == CP_K_BWD_FUSED)
        return attn_bwd_impl(problem, plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, stream,
                             kernel);
    return CP_ERR_INVALID_ARG;
}

// ---------------------------------------------------------------------------
// cp_attn_bwd_noalloc: the backward with its per-row scratch (dot(dO, O) and
// -LSE * log2(e), fp32 each) in a fixed device array instead of a caller
// workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoallocScratchBytes = size_t(2) * CP_NOALLOC_MAX_ROWS * sizeof(float);  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// The name g_noalloc_scratch is only a host-side handle; kernels need the
// device address.  It is looked up on every call made outside a stream capture
// (so a context re-created after cudaDeviceReset gets its own address) and
// cached per device for calls made while `stream` is being captured, where the
// lookup is not made.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

cp_status_t noalloc_scratch(cudaStream_t stream, void** out)
{
    const int dev = current_device();
    if (dev < 0) return CP_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return CP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone || !g_noalloc_ptr[dev]) {
        if (cap != cudaStreamCaptureStatusNone) return CP_ERR_CUDA;   // never looked up before capture
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CP_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return CP_OK;
}

}  // namespace

extern "C" cp_status_t cp_attn_bwd_noalloc(const cp_problem_t* problem, const cp_plan_t* plan,
                                           const void* q, const void* k, const void* v,
                                           const void* o, const float* lse, const void* dout,
                                           void* dq, void* dk, void* dv, void* stream)
{
    cp_status_t st = check_attention(problem);
    if (st != CP_OK) return st;
    if ((st = check_plan(plan, false, problem)) != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * problem->seq_len;
    if (rows > CP_NOALLOC_MAX_ROWS) return CP_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    void* scratch = nullptr;
    if ((st = noalloc_scratch(s, &scratch)) != CP_OK) return st;
    float* delta = static_cast<float*>(scratch);
    float* nlse2 = delta + CP_NOALLOC_MAX_ROWS;   // 16 MiB further: 256-byte aligned
    return launch_bwd_any(problem, plan, q, k, v, o, lse, dout, dq, dk, dv, delta, nlse2, s, 0, whole_layout(problem), nullptr, nullptr, nullptr);
}

// ---------------------------------------------------------------------------
// Per-rank entry points: context parallelism across GPUs, one process per GPU.
// Each rank holds its local query shard (Q_r, O_r, dO_r, dQ_r: 2C rows per
// head) and receives the K/V shards from the others (all-gather, or one shard
// per ring step); the backward's dK/dV contributions of every rank are summed
// across ranks by the caller (reduce-scatter) and cast with cp_f32_to_bf16.
// ---------------------------------------------------------------------------
namespace {

cp_status_t check_rank_call(const cp_problem_t* p, const cp_plan_t* pl, int32_t rank, int32_t step,
                            bool need_step)
{
    cp_status_t st = check_attention(p);
    if (st != CP_OK) return st;
    if ((st = check_plan(pl, false)) != CP_OK) return st;
    if (rank < 0 || rank >= p->cp_size) return CP_ERR_INVALID_ARG;
    if (need_step ? (step < 0 || step >= p->cp_size) : step != -1) return CP_ERR_INVALID_ARG;
    return CP_OK;
}

__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ in,
                                                          uint2* __restrict__ out, int64_t n4)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 x = __ldg(in + i);
        out[i] = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
    }
}

}  // namespace

extern "C" cp_status_t cp_attn_fwd_rank(const cp_problem_t* problem, const cp_plan_t* plan,
                                        int32_t rank, const void* q, const void* k, const void* v,
                                        void* o, float* lse, void* ws, size_t* ws_bytes, void* stream)
{
    cp_status_t st = check_rank_call(problem, plan, rank, -1, false);
    if (st != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    const int n2c = problem->seq_len / problem->cp_size;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * n2c;
    const bool separate = problem->merge == CP_MERGE_SEPARATE;
    const size_t o_parts_bytes = separate ? round_up(size_t(problem->cp_size) * rows * problem->head_dim * 4, 256) : 0;
    const size_t lse_parts_bytes = separate ? round_up(size_t(problem->cp_size) * rows * 4, 256) : 0;
    if (workspace_gate(o_parts_bytes + lse_parts_bytes, ws, ws_bytes, &st)) return st;
    float* o_parts = separate ? static_cast<float*>(ws) : nullptr;
    float* lse_parts = separate ? reinterpret_cast<float*>(static_cast<char*>(ws) + o_parts_bytes) : nullptr;
    cudaStream_t s = as_stream(stream);
    const Layout L = rank_layout(problem, rank, -1);
    st = launch_fwd_any(problem, plan, q, k, v, o, lse, o_parts, lse_parts, s, 0, L, !separate);
    if (st != CP_OK || !separate) return st;
    return launch_merge(rows, problem->head_dim, problem->cp_size, o_parts, lse_parts, o, lse, s, true);
}

extern "C" cp_status_t cp_attn_fwd_step(const cp_problem_t* problem, const cp_plan_t* plan,
                                        int32_t rank, int32_t step, const void* q, const void* k,
                                        const void* v, float* o_part, float* lse_part, void* stream)
{
    cp_status_t st = check_rank_call(problem, plan, rank, step, true);
    if (st != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o_part, lse_part};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const Layout L = rank_layout(problem, rank, step);
    return launch_fwd_any(problem, plan, q, k, v, nullptr, nullptr, o_part, lse_part, s, 0, L, false);
}

extern "C" cp_status_t cp_attn_bwd_rank(const cp_problem_t* problem, const cp_plan_t* plan,
                                        int32_t rank, const void* q, const void* k, const void* v,
                                        const void* o, const float* lse, const void* dout, void* dq,
                                        float* dk_part, float* dv_part, void* ws, size_t* ws_bytes,
                                        void* stream)
{
    cp_status_t st = check_rank_call(problem, plan, rank, -1, false);
    if (st != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk_part, dv_part};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    const int n2c = problem->seq_len / problem->cp_size;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * n2c;
    const size_t row_bytes = round_up(size_t(rows) * 4, 256);
    if (workspace_gate(2 * row_bytes, ws, ws_bytes, &st)) return st;
    float* delta = static_cast<float*>(ws);
    float* nlse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + row_bytes);
    cudaStream_t s = as_stream(stream);
    const Layout L = rank_layout(problem, rank, -1);
    return launch_bwd_any(problem, plan, q, k, v, o, lse, dout, dq, nullptr, nullptr, delta, nlse2, s, 0, L, dk_part, dv_part, nullptr);
}

extern "C" cp_status_t cp_attn_bwd_step(const cp_problem_t* problem, const cp_plan_t* plan,
                                        int32_t rank, int32_t step, const void* q, const void* k,
                                        const void* v, const void* o, const float* lse,
                                        const void* dout, float* dq_sum, float* dk_sum, float* dv_sum,
                                        void* ws, size_t* ws_bytes, void* stream)
{
    cp_status_t st = check_rank_call(problem, plan, rank, step, true);
    if (st != CP_OK) return st;
    const void* ptrs[] = {q, k, v, o, lse, dout, dq_sum, dk_sum, dv_sum};
    for (const void* x : ptrs)
        if (!x || !aligned16(x)) return CP_ERR_INVALID_ARG;
    const int n2c = problem->seq_len / problem->cp_size;
    const int64_t rows = static_cast<int64_t>(problem->batch) * problem->num_heads * n2c;
    const size_t row_bytes = round_up(size_t(rows) * 4, 256);
    if (workspace_gate(2 * row_bytes, ws, ws_bytes, &st)) return st;
    float* delta = static_cast<float*>(ws);
    float* nlse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + row_bytes);
    cudaStream_t s = as_stream(stream);
    const Layout L = rank_layout(problem, rank, step);   // rank r's rows, the one shard of the step
    return launch_bwd_any(problem, plan, q, k, v, o, lse, dout, nullptr, nullptr, nullptr, delta, nlse2, s, 0,
                          L, dk_sum, dv_sum, nullptr, dq_sum, true);
}

extern "C" cp_status_t cp_f32_to_bf16(const float* in, void* out, int64_t n, void* stream)
{
    if (n < 0 || n % 4 != 0) return CP_ERR_INVALID_ARG;
    if (n == 0) return CP_OK;
    if (!in || !out || !aligned16(in) || (reinterpret_cast<uintptr_t>(out) & 7u)) return CP_ERR_INVALID_ARG;
    const int64_t n4 = n / 4;
    const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, int64_t(num_sms()) * 8);
    cudaStream_t s = as_stream(stream);
    LaunchScope ls(CP_K_CAST, s);
    f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(reinterpret_cast<const float4*>(in),
                                                                   static_cast<uint2*>(out), n4);
    return launch_status();
}
