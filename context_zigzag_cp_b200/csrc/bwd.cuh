// Backward kernels.  Gradients of causal (optionally packed-document, optionally
// sliding-window) attention from the saved final LSE, with P = exp(scale q.k -
// LSE_q) recomputed on the fly:  D_q = dO_q . O_q,  dV_k = sum_q P dO_q,
// dS = P (dO_q . v_k - D_q),  dQ_q = scale sum_k dS k_k,  dK_k = scale sum_q dS q_q.
//
// Two deterministic passes, no atomics:
//   * bwd_prep_kernel: D (fp32) and -LSE * log2(e) per row.
//   * cp_bwd_dkdv_kernel (KV-tile major): a CTA takes a zigzag pair of 128-key
//     tiles of one KV head and, for each, visits every query head of its group
//     and every virtual rank's query tile that attends to it (the single-GPU
//     form of handing dK_j / dV_j back around the ring), accumulating dK and dV
//     in tensor memory:  S^T = K Q^T,  dP^T = V dO^T  ->  P^T, dS^T (bf16,
//     written into the dP^T columns)  ->  dV += P^T dO,  dK += dS^T Q.
//   * cp_bwd_dq_kernel (query-tile major, visiting the K/V shards in the plan's
//     order like the forward; Q and dO rows held in tensor memory):  S = Q K^T,
//     dP = dO V^T  ->  dS (bf16, shared memory)  ->  dQ += dS K.
// In both passes the elementwise step runs on four warpgroups (a thread owns
// one TMEM lane = one row), each taking 16 columns of each 64-column slice of
// the 128 score columns.  The warps copy their scores out of tensor memory and
// release it at once, so the MMA warp computes the next tile's scores while
// this tile's elementwise step runs; all four warpgroups finish slice 0 before
// slice 1, and the MMA warp issues slice 0's products (a 64-deep part of the K
// dimension) while slice 1 is computed.
// Each 128-row tile lives in one zigzag chunk, so original positions are
// linear inside a tile and the causal / document / window tests are per-tile
// ranges.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "zigzag.cuh"
#include "fwd.cuh"
#include "plan.cuh"

namespace cpattn {

// ----------------------------------------------------------------------------
// Preprocess: delta[row] = sum_d dO*O, nlse2[row] = -LSE * log2(e), and (for the
// one-pass backward) the row of the fp32 dQ accumulator set to zero.  A row is
// D/8 lanes of one warp, each reading 16 bytes (8 bf16) of O and of dO, so a
// warp covers 32*8/D rows per step with full 16-byte accesses (D = 64, 128 or 256).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                const float* __restrict__ lse, float* __restrict__ delta,
                float* __restrict__ nlse2, int64_t rows, int D, float* __restrict__ dq_acc)
{
    const int lane = threadIdx.x & 31;
    const int lpr = D / 8;                      // lanes per row
    const int rpw = 32 / lpr;                   // rows per warp step
    const int sub = lane / lpr, e = lane - sub * lpr;
    const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t base = warp_g * rpw; base < rows; base += nwarps * rpw) {
        const int64_t row = base + sub;
        float acc = 0.f;
        if (row < rows) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + e);
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + e);
            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 x = __bfloat1622float2(a2[i]), y = __bfloat1622float2(b2[i]);
                acc = fmaf(x.x, y.x, acc);
                acc = fmaf(x.y, y.y, acc);
            }
            if (dq_acc) {
                float4* z = reinterpret_cast<float4*>(dq_acc + row * D) + 2 * e;
                z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        // sum over the row's lpr lanes (a power of two, aligned inside the warp)
        for (int off = lpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (e == 0 && row < rows) {
            delta[row] = acc;
            nlse2[row] = __ldg(lse + row) * -1.4426950408889634f;
        }
    }
}

struct BwdParams {
    int32_t B, Hq, Hkv, S, cp, C;
    int32_t docs;
    int32_t wm1;             // sliding window - 1 (larger than S: no window)
    int32_t nc;              // last visible key of query q is q + nc: 0 causal, S none
    float scale;             // softmax scale
    float scale_log2;        // softmax scale * log2(e)
    int32_t n_items;
    int32_t stall;           // test hook: the cp_kernel_t whose CTA 0 skips its first K/V load
    // Row layouts (as in FwdParams): Q, dO, dQ and the per-row workspace hold q_rows
    // rows per batch*head starting at shard position q_base; K, V hold kv_rows rows
    // per batch*KV head starting at kv_base (-1: only the shard visited, 2C rows).
    // dK / dV cover all S keys, or with step_shard the visited shard's 2C keys.
    int32_t q_rows, q_base, kv_rows, kv_base;
    int32_t rank;            // -1: every rank's query rows; r: only rank r's
    int32_t s0, s1;          // dQ pass: visit steps s0 .. s1-1 (0 .. cp: the whole visit)
    int32_t step_shard;      // 1: the dK/dV pass covers only the shard rank `rank` visits at step s0
    int32_t accumulate;      // 1: dq32 / dk32 / dv32 are fp32 sums that the pass adds into
    float* dq32;             // non-null: dQ (scaled) in fp32 here instead of bf16 in dq
    float* dk32;             // non-null: dK / dV written as fp32 partials here instead of bf16
    float* dv32;
    float* dq_acc;           // one-pass backward: fp32 dQ accumulator [B*Hq][q_rows][D] (unscaled)
    const int32_t* tile_orig;   // per-document plans (as in FwdParams); null otherwise
    const int32_t* tile_shard;
    const int32_t* src;      // [cp*cp]
    const int32_t* doc_start;  // [S] shard order
    const int32_t* cu;       // [num_docs+1] document offsets, original order (documents only)
    int32_t num_docs;
    const float* nlse2;      // [B*Hq][S], -LSE * log2(e)
    const float* delta;      // [B*Hq][S]
    const __nv_bfloat16* q;  // [B*Hq][S][D]
    const __nv_bfloat16* dout;  // [B*Hq][S][D]
    __nv_bfloat16* dq;       // [B*Hq][S][D]
    __nv_bfloat16* dk;       // [B*Hkv][S][D]
    __nv_bfloat16* dv;
};

// Of every four column pairs in the dK/dV pass's P, this many take 2^x from
// the FMA-pipe polynomial (exp2_poly.cuh) instead of ex2.approx.  Measured on
// B200 (gqa32k / long128k): 0 of 4 is fastest (1 and 2 of 4 cost 2-4 %), so
// the elementwise step is not bound by the special-function pipe.
#ifndef CP_BWD_POLY_PAIRS
#define CP_BWD_POLY_PAIRS 0
#endif

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^x for a pair: ex2.approx, or the polynomial when poly (a constant once the
// caller's loop is unrolled).
__device__ __forceinline__ uint64_t exp2_pair(uint64_t x2, bool poly)
{
    if (poly) return exp2_poly2(x2);
    float a, b;
    f2_unpack(x2, a, b);
    return f2_pack(ex2_approx(a), ex2_approx(b));
}

// P^T for 16 query columns of one key row k in the dK/dV pass, in place over
// the scores: P = 2^(s * scale * log2(e) - LSE * log2(e)).  MODE 0: every
// column admitted; 1: column c admitted when thr <= c <= thr + wm1 (thr = k -
// first query of the 16: the causal test and the sliding window); 2: also
// k >= ds[c] (documents).
template <int MODE>
__device__ __forceinline__ void dkdv_p16(float* sv, const float* s_nlse2, const int* s_ds, float scale_log2,
                                         int thr, int wm1, int k_orig)
{
    const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        const uint2 l01 = *reinterpret_cast<const uint2*>(s_nlse2 + i);
        const uint2 l23 = *reinterpret_cast<const uint2*>(s_nlse2 + i + 2);
        const uint64_t x01 = f2_fma(f2_pack(sv[i], sv[i + 1]), sc2,
                                    (static_cast<uint64_t>(l01.y) << 32) | l01.x);
        const uint64_t x23 = f2_fma(f2_pack(sv[i + 2], sv[i + 3]), sc2,
                                    (static_cast<uint64_t>(l23.y) << 32) | l23.x);
        // pairs i/2 and i/2 + 1; pair k takes the polynomial when k % 4 < CP_BWD_POLY_PAIRS
        const uint64_t p01 = exp2_pair(x01, ((i / 2) % 4) < CP_BWD_POLY_PAIRS);
        const uint64_t p23 = exp2_pair(x23, ((i / 2 + 1) % 4) < CP_BWD_POLY_PAIRS);
        float p4[4];
        f2_unpack(p01, p4[0], p4[1]);
        f2_unpack(p23, p4[2], p4[3]);
        int dsv[4] = {0, 0, 0, 0};
        if (MODE == 2) {
            const int4 q4 = *reinterpret_cast<const int4*>(s_ds + i);
            dsv[0] = q4.x; dsv[1] = q4.y; dsv[2] = q4.z; dsv[3] = q4.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (MODE >= 1 && (i + e < thr || i + e > thr + wm1)) p4[e] = 0.f;
            if (MODE == 2 && k_orig < dsv[e]) p4[e] = 0.f;
            sv[i + e] = p4[e];
        }
    }
}

// dS^T = P^T (dP^T - delta) for 16 query columns, and both packed to bf16 pairs.
__device__ __forceinline__ void dkdv_ds16(const float* pv, const float* dp, const float* s_delta, uint32_t* pk,
                                          uint32_t* dk)
{
    const uint64_t m1 = f2_pack(-1.f, -1.f);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const uint2 d2 = *reinterpret_cast<const uint2*>(s_delta + i);
        const uint64_t p2 = f2_pack(pv[i], pv[i + 1]);
        const uint64_t g2 = f2_mul(p2, f2_fma((static_cast<uint64_t>(d2.y) << 32) | d2.x, m1,
                                              f2_pack(dp[i], dp[i + 1])));
        float g0, g1;
        f2_unpack(g2, g0, g1);
        pk[i / 2] = pack_bf16(pv[i], pv[i + 1]);
        dk[i / 2] = pack_bf16(g0, g1);
    }
}

// P for 16 key columns of one query row in the dQ pass, in place over the
// scores, with packed f32x2 arithmetic; with MASK, column c is admitted when
// lo <= c <= hi.
template <bool MASK>
__device__ __forceinline__ void dq_p16(float* sv, float nlse2, float scale_log2, int lo, int hi)
{
    const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nl2 = f2_pack(nlse2, nlse2);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float a, b;
        f2_unpack(f2_fma(f2_pack(sv[i], sv[i + 1]), sc2, nl2), a, b);
        a = ex2_approx(a);
        b = ex2_approx(b);
        if (MASK) {
            if (i < lo || i > hi) a = 0.f;
            if (i + 1 < lo || i + 1 > hi) b = 0.f;
        }
        sv[i] = a;
        sv[i + 1] = b;
    }
}

// dS = P (dP - delta) for 16 key columns, packed to bf16 pairs.
__device__ __forceinline__ void dq_ds16(const float* pv, const float* dp, float dlt, uint32_t* dk)
{
    const uint64_t nd2 = f2_pack(-dlt, -dlt);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float a, b;
        f2_unpack(f2_mul(f2_pack(pv[i], pv[i + 1]), f2_add(f2_pack(dp[i], dp[i + 1]), nd2)), a, b);
        dk[i / 2] = pack_bf16(a, b);
    }
}

// ============================================================================
// dK / dV pass
// ============================================================================
// One past the last query tile that can attend to the key tile at original ko:
// queries come at or after the key under the causal mask (the loop starts at
// tile (ko - nc) / 128, ko's own tile when causal, tile 0 when not), no later than
// the window allows, and inside the document of the tile's last key.
__device__ __forceinline__ int dkdv_last_tile(const BwdParams& P, int ko, int ntq)
{
    int t_end = min(ntq, (ko + 127 + P.wm1) / 128 + 1);
    if (P.docs) {
        const int de = __ldg(P.cu + doc_index(P.cu, P.num_docs, ko + 127) + 1);
        t_end = min(t_end, (de - 1) / 128 + 1);
    }
    return t_end;
}
// The order in which a work unit's half visits its key tile's query tiles
// [t0, t1): u runs over [u0, u1) and the query tile is |u|.  The first half's key
// tile (attended by the long run of query tiles from its own position to the end)
// walks them from the end down (u from 1 - t1 to -t0), the second half's (the
// short run at the end) upwards (u = t).  Every CTA of a wave starts its two halves
// at the same times, so at any moment the first halves all read one query tile
// and the second halves another, each from L2 after its first reader; walked
// upwards, the first halves would read a window as wide as the wave.
struct DkdvWalk {
    int u0, u1;
};
__device__ __forceinline__ DkdvWalk dkdv_walk(int t0, int t1, int iter)
{
    return (iter & 1) ? DkdvWalk{t0, t1} : DkdvWalk{1 - t1, 1 - t0};
}
// True when the query tile at shard position qpos belongs to the rank the pass
// runs for (always, for a whole-sequence pass).
__device__ __forceinline__ bool q_tile_on_rank(const BwdParams& P, int qpos)
{
    return P.rank < 0 || qpos / (2 * P.C) == P.rank;
}

constexpr int BWD_NWG = 4;                       // elementwise warpgroups
constexpr int BWD_THREADS = (BWD_NWG + 1) * 128; // + producer / MMA warpgroup
constexpr int BWD_NSLICE = 2;                    // 64-column slices of a 128-column score tile

template <int D>
struct DkdvCfg {
    static constexpr int TILE = 128 * D * 2;
    // Q tiles are needed early (S^T of the next tile is issued while the current one is
    // still in the elementwise step), dO tiles later: three Q slots, each with the tile's
    // nlse2 row (512 B, used with S^T), and two dO slots, each with its delta row.
    static constexpr int NQ = 3, NDO = 2;
    static constexpr int K_OFF = 0, V_OFF = TILE;
    static constexpr int Q_OFF = 2 * TILE;
    static constexpr int DO_OFF = Q_OFF + NQ * TILE;
    static constexpr int LQ_OFF = DO_OFF + NDO * TILE;           // nlse2 rows [NQ]
    static constexpr int LD_OFF = LQ_OFF + NQ * 512;              // delta rows [NDO]
    static constexpr int BAR_OFF = LD_OFF + NDO * 512;
    // kv_full, kv_empty, q_full[NQ], q_empty[NQ], do_full[NDO], do_empty[NDO], st_ready, dp_ready,
    // s_free, (a spare slot), p_full[NSLICE], acc_full, drain, acc_empty
    static constexpr int NBAR = 9 + 2 * NQ + 2 * NDO + BWD_NSLICE;
    // the dynamic shared window starts 1024-byte aligned (checked at run time), no slack
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64;
    static constexpr int THREADS = BWD_THREADS;
};

struct DkdvItem {
    int bkv, b, hk, kpos, ko;
    int krow;                // the key tile's first row in K / V (and, with step_shard, in dK / dV)
};

// A work unit is a pair of key tiles of one KV head, original tiles p and
// nkt - 1 - p (the backward's form of the zigzag pairing): under the causal
// mask the pair attends to nkt + 1 query tiles whatever p is, so every CTA
// gets the same work.  A CTA takes unit blockIdx.x + i * gridDim.x and does its
// two key tiles one after the other (half 0, then half 1); for each it visits
// the attending query tiles by ascending original position.  The CTAs of one
// wave then read query tiles that lie within a window of about gridDim.x tiles
// (first halves) or are the same tile (second halves), so each query tile comes
// from DRAM about once per wave instead of once per CTA.
template <bool PD>
__device__ __forceinline__ DkdvItem decode_dkdv(const BwdParams& P, int unit, int half)
{
    DkdvItem it;
    // with step_shard, the tiles of the one shard visited (zigzag pairs inside it)
    const int nkt = P.step_shard ? 2 * P.C / 128 : P.S / 128;
    const int npair = nkt / 2;
    it.bkv = unit / npair;
    const int pidx = unit - it.bkv * npair;
    const int t = half ? nkt - 1 - pidx : pidx;
    it.b = it.bkv / P.Hkv;
    it.hk = it.bkv - it.b * P.Hkv;
    if (P.step_shard) {
        const int j = __ldg(P.src + P.rank * P.cp + P.s0);
        it.ko = tile_orig_of<PD>(P, j, t, P.C / 128);
        it.kpos = j * 2 * P.C + t * 128;
        it.krow = t * 128;
    } else {
        it.ko = t * 128;
        it.kpos = shard_of_tile<PD>(P, it.ko);
        it.krow = it.kpos - P.kv_base;
    }
    return it;
}

template <int D, bool PD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
cp_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const BwdParams P)
{
    using Cfg = DkdvCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023u) {   // swizzled tiles need a 1024-byte aligned window
        if (threadIdx.x == 0) record_status(3 /* CP_ERR_CUDA */);
        return;
    }
    uint8_t* smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sK = sbase + Cfg::K_OFF, sV = sbase + Cfg::V_OFF;
    const uint32_t sQ = sbase + Cfg::Q_OFF, sdO = sbase + Cfg::DO_OFF;
    const uint32_t sLQ = sbase + Cfg::LQ_OFF, sLD = sbase + Cfg::LD_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_kv_full = bars, bar_kv_empty = bars + 8;
    const uint32_t bar_q_full = bars + 16, bar_q_empty = bar_q_full + 8 * Cfg::NQ;
    const uint32_t bar_do_full = bar_q_empty + 8 * Cfg::NQ, bar_do_empty = bar_do_full + 8 * Cfg::NDO;
    const uint32_t bar_st_ready = bar_do_empty + 8 * Cfg::NDO, bar_dp_ready = bar_st_ready + 8;
    const uint32_t bar_s_free = bar_dp_ready + 8;
    const uint32_t bar_p_full = bar_s_free + 16;                      // [NSLICE]
    const uint32_t bar_acc_full = bar_p_full + 8 * BWD_NSLICE, bar_drain = bar_acc_full + 8;
    const uint32_t bar_acc_empty = bar_drain + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8 + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.Hq / P.Hkv;
    const int ntq = P.S / 128;                 // query tiles, visited by ascending original position
    constexpr int PROD_WARP = 4 * BWD_NWG, MMA_WARP = 4 * BWD_NWG + 1;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar_kv_full, 1);
        mbar_init(bar_kv_empty, 1);
        for (int i = 0; i < Cfg::NQ; ++i) {
            mbar_init(bar_q_full + 8 * i, 1);
            mbar_init(bar_q_empty + 8 * i, 1);
        }
        for (int i = 0; i < Cfg::NDO; ++i) {
            mbar_init(bar_do_full + 8 * i, 1);
            mbar_init(bar_do_empty + 8 * i, 1);
        }
        mbar_init(bar_st_ready, 1);
        mbar_init(bar_dp_ready, 1);
        mbar_init(bar_s_free, 4 * BWD_NWG);
        for (int i = 0; i < BWD_NSLICE; ++i) mbar_init(bar_p_full + 8 * i, 4 * BWD_NWG);
        mbar_init(bar_acc_full, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_acc_empty, 4 * BWD_NWG);
        fence_barrier_init();
    }
    if (warp == MMA_WARP) tmem_alloc(smem_u32(tmem_slot), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 4 * BWD_NWG) {
      // producer / MMA warpgroup gives registers to the elementwise groups
      // (4*128*104 + 128*64 = 640*96, the block's launch allotment)
      regs_dec<64>();
      if (warp == PROD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmdO);
            uint32_t nst = 0, iter = 0;
            bool ok = true, kv_issued = false;
            for (int w = blockIdx.x; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
                const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
                ok = mbar_wait(bar_kv_empty, (iter & 1) ^ 1, abort_flag);
                if (!ok) break;
                kv_issued = true;
                // test hook (cp_selftest_stall): the first K/V tile of CTA 0 is never loaded
                if (!(P.stall == 7 /* CP_K_BWD_DKDV */ && blockIdx.x == 0 && iter == 0)) {
                    mbar_arrive_expect_tx(bar_kv_full, 2 * Cfg::TILE);
                    for (int h = 0; h < D / 64; ++h) {
                        const int kvrow = it.bkv * P.kv_rows + it.krow;
                        tma_load_2d(sK + h * 16384, &tmK, h * 64, kvrow, bar_kv_full);
                        tma_load_2d(sV + h * 16384, &tmV, h * 64, kvrow, bar_kv_full);
                    }
                }
                const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
                for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                    const int qo = abs(u) * 128;
                    const int qpos = shard_of_tile<PD>(P, qo);
                    const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                    const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 127) : 0, qo + 127 - P.wm1);
                    if (classify_tile(qo, dsf, dsl, it.ko, P.nc) == TILE_SKIP || !q_tile_on_rank(P, qpos))
                        continue;
                    for (int hq = 0; hq < g && ok; ++hq) {
                        const int bh = it.b * P.Hq + it.hk * g + hq;
                        const size_t row = static_cast<size_t>(bh) * P.q_rows + (qpos - P.q_base);
                        const uint32_t qs = nst % Cfg::NQ, qp = (nst / Cfg::NQ) & 1;
                        const uint32_t ds = nst % Cfg::NDO, dpar = (nst / Cfg::NDO) & 1;
                        ++nst;
                        ok = mbar_wait(bar_q_empty + 8 * qs, qp ^ 1, abort_flag);
                        if (!ok) break;
                        mbar_arrive_expect_tx(bar_q_full + 8 * qs, Cfg::TILE + 512);
                        for (int h = 0; h < D / 64; ++h)
                            tma_load_2d(sQ + qs * Cfg::TILE + h * 16384, &tmQ, h * 64, static_cast<int>(row),
                                        bar_q_full + 8 * qs);
                        bulk_load(sLQ + qs * 512, P.nlse2 + row, 512, bar_q_full + 8 * qs);
                        ok = mbar_wait(bar_do_empty + 8 * ds, dpar ^ 1, abort_flag);
                        if (!ok) break;
                        mbar_arrive_expect_tx(bar_do_full + 8 * ds, Cfg::TILE + 512);
                        for (int h = 0; h < D / 64; ++h)
                            tma_load_2d(sdO + ds * Cfg::TILE + h * 16384, &tmdO, h * 64, static_cast<int>(row),
                                        bar_do_full + 8 * ds);
                        bulk_load(sLD + ds * 512, P.delta + row, 512, bar_do_full + 8 * ds);
                    }
                }
            }
            if (!ok) {   // let the copies in flight land before the CTA exits (bounded waits)
                for (uint32_t n = (nst > Cfg::NQ ? nst - Cfg::NQ : 0); n < nst; ++n)
                    mbar_wait_drain(bar_q_full + 8 * (n % Cfg::NQ), (n / Cfg::NQ) & 1);
                for (uint32_t n = (nst > Cfg::NDO ? nst - Cfg::NDO : 0); n < nst; ++n)
                    mbar_wait_drain(bar_do_full + 8 * (n % Cfg::NDO), (n / Cfg::NDO) & 1);
                if (kv_issued) mbar_wait_drain(bar_kv_full, (iter & 1));
            }
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the control flow; one elected lane issues each group
        // of tensor-core instructions (cheaper than a single diverged lane).
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);   // K-major A and B
            constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);      // A tmem, B MN-major
            constexpr uint32_t TILE16 = Cfg::TILE >> 4;
            const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
            // descriptor bases; k-steps and stages are constant offsets in 16-byte units
            const uint64_t dK = sdesc_sw128(sK, 16, 1024), dVk = sdesc_sw128(sV, 16, 1024);
            const uint64_t dQk = sdesc_sw128(sQ, 16, 1024), dQmn = sdesc_sw128(sQ, 16384, 1024);
            const uint64_t dOk = sdesc_sw128(sdO, 16, 1024), dOmn = sdesc_sw128(sdO, 16384, 1024);
            uint32_t nst = 0, iter = 0, sf_phase = 0, ae_phase = 0;
            uint32_t p_phase[BWD_NSLICE];
            for (int i = 0; i < BWD_NSLICE; ++i) p_phase[i] = 0;
            // acc_busy: the last item's accumulators not yet read out; s_pending: S^T / dP^T of the
            // last issued tile not yet copied out by the elementwise warps
            bool ok = true, acc_busy = false, s_pending = false;
            // dV += P^T dO, dK += dS^T Q for one finished query tile.  P^T and dS^T (bf16) sit in
            // the dP^T columns: query rows 64j + 16w .. +15 of slice j at 64j + 16w (P^T) and
            // 64j + 16w + 8 (dS^T), each warp's over the 16 columns of dP^T it read.
            auto issue_products = [&](uint32_t qs, uint32_t ds, bool& first) -> bool {
                if (first && acc_busy) {   // every group has stored the previous item's dK / dV
                    if (!mbar_wait_warp(bar_acc_empty, ae_phase, abort_flag)) return false;
                    ae_phase ^= 1;
                    acc_busy = false;
                }
                const uint64_t bq_mn = dQmn + qs * TILE16, bdo_mn = dOmn + ds * TILE16;
                for (int j = 0; j < BWD_NSLICE; ++j) {
                    if (!mbar_wait_warp(bar_p_full + 8 * j, p_phase[j], abort_flag)) return false;
                    p_phase[j] ^= 1;
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) {
                            const uint32_t acc = (!first || j > 0 || w4 > 0) ? 1u : 0u;
                            const uint32_t brow = ((4 * j + w4) * 2048) >> 4;
                            mma_ts(tdV, tdP + 64 * j + 16 * w4, bdo_mn + brow, IDESC_G, acc);
                            mma_ts(tdK, tdP + 64 * j + 16 * w4 + 8, bq_mn + brow, IDESC_G, acc);
                        }
                    }
                    __syncwarp();
                }
                first = false;
                if (elect_one()) {
                    mma_commit(bar_q_empty + 8 * qs);
                    mma_commit(bar_do_empty + 8 * ds);
                }
                __syncwarp();
                return true;
            };
            for (int w = blockIdx.x; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
                const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
                ok = mbar_wait_warp(bar_kv_full, iter & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool first = true, prev_live = false;
                uint32_t prev_qs = 0, prev_ds = 0;
                const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
                for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                    const int qo = abs(u) * 128;
                    const int qpos = shard_of_tile<PD>(P, qo);
                    const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                    const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 127) : 0, qo + 127 - P.wm1);
                    if (classify_tile(qo, dsf, dsl, it.ko, P.nc) == TILE_SKIP || !q_tile_on_rank(P, qpos))
                        continue;
                    for (int hq = 0; hq < g && ok; ++hq) {
                        const uint32_t qs = nst % Cfg::NQ, qp = (nst / Cfg::NQ) & 1;
                        const uint32_t ds = nst % Cfg::NDO, dpar = (nst / Cfg::NDO) & 1;
                        ++nst;
                        ok = mbar_wait_warp(bar_q_full + 8 * qs, qp, abort_flag);
                        if (!ok) break;
                        if (s_pending) {   // the previous tile's S^T / dP^T are copied out
                            ok = mbar_wait_warp(bar_s_free, sf_phase, abort_flag);
                            if (!ok) break;
                            sf_phase ^= 1;
                        }
                        tc_fence_after();
                        const uint64_t bq = dQk + qs * TILE16, bdo = dOk + ds * TILE16;
                        // S^T of this tile while the elementwise warps still work on the previous one
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ss(tS, dK + off, bq + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_st_ready);
                        }
                        __syncwarp();
                        // the previous tile's products read P^T / dS^T from the dP^T columns ...
                        if (prev_live && !(ok = issue_products(prev_qs, prev_ds, first))) break;
                        ok = mbar_wait_warp(bar_do_full + 8 * ds, dpar, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        // ... before this tile's dP^T overwrites them (the tensor pipe runs in order)
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ss(tdP, dVk + off, bdo + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_dp_ready);
                        }
                        __syncwarp();
                        s_pending = true;
                        prev_live = true;
                        prev_qs = qs;
                        prev_ds = ds;
                    }
                }
                if (ok && prev_live) ok = issue_products(prev_qs, prev_ds, first);
                if (!ok) break;
                if (elect_one()) {
                    mma_commit(bar_kv_empty);
                    if (!first) mma_commit(bar_acc_full);   // the elementwise groups wait only if they had a tile
                }
                __syncwarp();
                acc_busy = acc_busy || !first;
            }
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            mbar_wait_drain(bar_drain, 0);
        }
      }
    } else {
        regs_inc<104>();
        // ------------------------------------------------------------ elementwise groups (key rows)
        const int wg = warp >> 2;                        // query columns [16wg, 16wg+16) of each slice
        const int row = (warp & 3) * 32 + lane;          // key row of the tile (TMEM lane)
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 16 * wg, tdP = tmem + lane_off + 128 + 16 * wg;
        const uint32_t tdV = tmem + lane_off + 256 + 32 * wg, tdK = tmem + lane_off + 384 + 32 * wg;
        // packed P^T / dS^T of slice j go to dP^T columns 64j + 8wg and 64j + 32 + 8wg
        // packed P^T / dS^T of slice j go over this warp's own dP^T columns, already read:
        // 64j + 16wg (P^T) and 64j + 16wg + 8 (dS^T)
        const uint32_t tPk = tmem + lane_off + 128 + 16 * wg, tDk = tPk + 8;
        uint32_t nst = 0, st_phase = 0, dp_phase = 0, a_phase = 0;
        bool ok = true;
        for (int w = blockIdx.x, iter = 0; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
            const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
            const int k_orig = it.ko + row;
            bool had = false;
            const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
            for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                const int qo = abs(u) * 128;
                const int qpos = shard_of_tile<PD>(P, qo);
                const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 127) : 0, qo + 127 - P.wm1);
                const int cls = classify_tile(qo, dsf, dsl, it.ko, P.nc);
                if (cls == TILE_SKIP || !q_tile_on_rank(P, qpos)) continue;
                for (int hq = 0; hq < g && ok; ++hq) {
                    const uint32_t qs = nst % Cfg::NQ, ds = nst % Cfg::NDO;
                    ++nst;
                    const float* s_nlse2 = reinterpret_cast<const float*>(smem + Cfg::LQ_OFF + qs * 512) + 16 * wg;
                    const float* s_delta = reinterpret_cast<const float*>(smem + Cfg::LD_OFF + ds * 512) + 16 * wg;
                    const int* s_ds = P.doc_start + qpos + 16 * wg;   // documents only (global, cached)
                    // ---- S^T: copy out, release, and form P^T while dP^T is still being computed
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_st_ready, st_phase, abort_flag));
                    if (!ok) break;
                    st_phase ^= 1;
                    tc_fence_after();
                    float sv[32], dp[32];
                    tmem_ld16f(tS, sv);
                    tmem_ld16f(tS + 64, sv + 16);
                    tmem_wait_ld();
                    reg_fence32f(sv);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_s_free);   // the MMA warp may compute the next S^T
#pragma unroll
                    for (int j = 0; j < BWD_NSLICE; ++j) {
                        // column c (query qo + 64j + 16wg + c) is admitted when k - nc <= q
                        // and q <= k + wm1: thr - nc <= c <= thr + wm1
                        const int thr = k_orig - (qo + 64 * j + 16 * wg) - P.nc;
                        const int wsp = P.wm1 + P.nc;
                        if (cls == TILE_FULL)
                            dkdv_p16<0>(sv + 16 * j, s_nlse2 + 64 * j, s_ds + 64 * j, P.scale_log2, thr, wsp, k_orig);
                        else if (!P.docs)
                            dkdv_p16<1>(sv + 16 * j, s_nlse2 + 64 * j, s_ds + 64 * j, P.scale_log2, thr, wsp, k_orig);
                        else
                            dkdv_p16<2>(sv + 16 * j, s_nlse2 + 64 * j, s_ds + 64 * j, P.scale_log2, thr, wsp, k_orig);
                    }
                    // ---- dP^T: copy out; the packed results go over this warp's own columns
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_ready, dp_phase, abort_flag));
                    if (!ok) break;
                    dp_phase ^= 1;
                    tc_fence_after();
                    tmem_ld16f(tdP, dp);
                    tmem_ld16f(tdP + 64, dp + 16);
                    tmem_wait_ld();
                    reg_fence32f(dp);
#pragma unroll
                    for (int j = 0; j < BWD_NSLICE; ++j) {
                        uint32_t pk[8], dk[8];
                        dkdv_ds16(sv + 16 * j, dp + 16 * j, s_delta + 64 * j, pk, dk);
                        tmem_st8(tPk + 64 * j, pk);
                        tmem_st8(tDk + 64 * j, dk);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_full + 8 * j);
                    }
                    had = true;
                }
            }
            if (!ok) break;
            // ---- epilogue: this group's 32 columns of dK (scaled) and dV
            const size_t orow = P.step_shard ? static_cast<size_t>(it.bkv) * 2 * P.C + it.krow + row
                                             : static_cast<size_t>(it.bkv) * P.S + it.kpos + row;
            if (had) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full, a_phase, abort_flag));
                if (!ok) break;
                a_phase ^= 1;
                tc_fence_after();
                if (32 * wg < D) {
                    float a[32], b[32];
                    tmem_ld32f(tdV, a);
                    tmem_ld32f(tdK, b);
                    tmem_wait_ld();
                    reg_fence32f(a);
                    reg_fence32f(b);
                    if (P.dk32) {   // fp32 partials (one rank's share, summed across ranks later)
                        float4* dv = reinterpret_cast<float4*>(P.dv32 + orow * D + 32 * wg);
                        float4* dk = reinterpret_cast<float4*>(P.dk32 + orow * D + 32 * wg);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float4 x = make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
                            float4 y = make_float4(b[4 * i] * P.scale, b[4 * i + 1] * P.scale,
                                                   b[4 * i + 2] * P.scale, b[4 * i + 3] * P.scale);
                            if (P.accumulate) {   // this CTA owns the rows: a plain read-modify-write
                                const float4 u = dv[i], w = dk[i];
                                x.x += u.x; x.y += u.y; x.z += u.z; x.w += u.w;
                                y.x += w.x; y.y += w.y; y.z += w.z; y.w += w.w;
                            }
                            dv[i] = x;
                            dk[i] = y;
                        }
                    } else {
                    uint4* dv = reinterpret_cast<uint4*>(P.dv + orow * D + 32 * wg);
                    uint4* dk = reinterpret_cast<uint4*>(P.dk + orow * D + 32 * wg);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        dv[i] = make_uint4(pack_bf16(a[8 * i], a[8 * i + 1]), pack_bf16(a[8 * i + 2], a[8 * i + 3]),
                                           pack_bf16(a[8 * i + 4], a[8 * i + 5]), pack_bf16(a[8 * i + 6], a[8 * i + 7]));
                        dk[i] = make_uint4(pack_bf16(b[8 * i] * P.scale, b[8 * i + 1] * P.scale),
                                           pack_bf16(b[8 * i + 2] * P.scale, b[8 * i + 3] * P.scale),
                                           pack_bf16(b[8 * i + 4] * P.scale, b[8 * i + 5] * P.scale),
                                           pack_bf16(b[8 * i + 6] * P.scale, b[8 * i + 7] * P.scale));
                    }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty);
            } else if (32 * wg < D && !P.accumulate) {
                if (P.dk32) {
                    float4* dv = reinterpret_cast<float4*>(P.dv32 + orow * D + 32 * wg);
                    float4* dk = reinterpret_cast<float4*>(P.dk32 + orow * D + 32 * wg);
                    for (int i = 0; i < 8; ++i) { dv[i] = make_float4(0.f, 0.f, 0.f, 0.f); dk[i] = dv[i]; }
                } else {
                    uint4* dv = reinterpret_cast<uint4*>(P.dv + orow * D + 32 * wg);
                    uint4* dk = reinterpret_cast<uint4*>(P.dk + orow * D + 32 * wg);
                    for (int i = 0; i < 4; ++i) { dv[i] = make_uint4(0, 0, 0, 0); dk[i] = make_uint4(0, 0, 0, 0); }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        __syncwarp();
        tc_fence_after();
        tmem_relinquish();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================================
// dQ pass
// ============================================================================
// The query tile's Q and dO rows sit in tensor memory (the A operands of S and
// dP, written by the elementwise warps once per item), so shared memory holds
// a deep K/V ring.  Same schedule as the dK/dV pass: the elementwise warps copy
// S out and release it (s_free), so the MMA warp computes the next key tile's S
// at once; they form P while the previous tile's products and this tile's dP
// are on the tensor core, copy dP out, and write dS (bf16) over the dP columns
// each warp has just read, in two 64-key slices; slice 0's
// dQ += dS K (A from tensor memory) runs while slice 1 is formed.
// Tensor memory: S 0..127, dP 128..255, dQ 256..383, Q 384..447, dO 448..511.
template <int D>
struct DqCfg {
    static constexpr int KTILE = 128 * D * 2;
    static constexpr int NSLOT = (D == 128) ? 6 : 12;
    static constexpr int KV_OFF = 0;
    static constexpr int BAR_OFF = KV_OFF + NSLOT * KTILE;
    // qt_full, qt_empty, kv_full[NSLOT], kv_empty[NSLOT], st_ready, dp_ready, s_free, (spare),
    // p_full[NSLICE], acc_full, drain, acc_empty
    static constexpr int NBAR = 9 + 2 * NSLOT + BWD_NSLICE;
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64 + 1024;
    static constexpr int THREADS = BWD_THREADS;
};

struct DqItem {
    int bh, bkv, r, qpos, qo;
};

// Items run GQA group by group; inside a group, query tiles by descending
// original position (the longest first) with the group's query heads fastest,
// so the CTAs in flight stream the same K/V tiles of one KV head.
template <bool PD>
__device__ __forceinline__ DqItem decode_dq(const BwdParams& P, int w)
{
    DqItem it;
    const int g = P.Hq / P.Hkv;
    const int ntiles = P.rank < 0 ? P.S / 128 : 2 * P.C / 128;   // every tile, or rank r's
    const int per_group = g * ntiles;
    it.bkv = w / per_group;
    const int rem = w - it.bkv * per_group;
    const int t = rem / g, hq = rem - t * g;
    const int b = it.bkv / P.Hkv, hk = it.bkv - b * P.Hkv;
    it.bh = b * P.Hq + hk * g + hq;
    if (P.rank < 0) {
        it.qo = (ntiles - 1 - t) * 128;      // descending original position
        it.qpos = shard_of_tile<PD>(P, it.qo);
    } else if (PD) {                         // rank r, per-document plan: its tiles, last first
        it.qpos = P.rank * 2 * P.C + (ntiles - 1 - t) * 128;
        it.qo = orig_of_tile<PD>(P, it.qpos);
    } else {                                 // rank r: its tail chunk, then its head chunk
        const int half = P.C / 128;
        it.qo = t < half ? (2 * P.cp - 1 - P.rank) * P.C + (half - 1 - t) * 128
                         : P.rank * P.C + (2 * half - 1 - t) * 128;
        it.qpos = shard_of_orig(it.qo, P.C, P.cp);
    }
    it.r = it.qpos / (2 * P.C);
    return it;
}

template <int D, bool PD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
cp_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams P)
{
    using Cfg = DqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sKV = sbase + Cfg::KV_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_qt_full = bars, bar_qt_empty = bars + 8;
    const uint32_t bar_kv_full = bars + 16, bar_kv_empty = bars + 16 + 8 * Cfg::NSLOT;
    const uint32_t bar_st_ready = bars + 16 + 16 * Cfg::NSLOT, bar_dp_ready = bar_st_ready + 8;
    const uint32_t bar_s_free = bar_dp_ready + 8;
    const uint32_t bar_p_full = bar_s_free + 16;                        // [NSLICE]
    const uint32_t bar_acc_full = bar_p_full + 8 * BWD_NSLICE, bar_drain = bar_acc_full + 8;
    const uint32_t bar_acc_empty = bar_drain + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8 + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n2c = 2 * P.C;
    const int half = P.C / 128;
    constexpr int PROD_WARP = 4 * BWD_NWG, MMA_WARP = 4 * BWD_NWG + 1;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar_qt_full, 4 * BWD_NWG);
        mbar_init(bar_qt_empty, 1);
        for (int i = 0; i < Cfg::NSLOT; ++i) {
            mbar_init(bar_kv_full + 8 * i, 1);
            mbar_init(bar_kv_empty + 8 * i, 1);
        }
        mbar_init(bar_st_ready, 1);
        mbar_init(bar_dp_ready, 1);
        mbar_init(bar_s_free, 4 * BWD_NWG);
        for (int i = 0; i < BWD_NSLICE; ++i) mbar_init(bar_p_full + 8 * i, 4 * BWD_NWG);
        mbar_init(bar_acc_full, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_acc_empty, 4 * BWD_NWG);
        fence_barrier_init();
    }
    if (warp == MMA_WARP) tmem_alloc(smem_u32(tmem_slot), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 4 * BWD_NWG) {
      // producer / MMA warpgroup gives registers to the elementwise groups
      // (4*128*104 + 128*64 = 640*96, the block's launch allotment)
      regs_dec<64>();
      if (warp == PROD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK); prefetch_tmap(&tmV);
            uint32_t nload = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x) {
                const DqItem it = decode_dq<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int kpos = j * n2c + kt * 128;
                        const int ko = tile_orig_of<PD>(P, j, kt, half);
                        if (classify_tile(it.qo, dsf, dsl, ko, P.nc) == TILE_SKIP) continue;
                        for (int kv = 0; kv < 2 && ok; ++kv, ++nload) {
                            const uint32_t slot = nload % Cfg::NSLOT, par = (nload / Cfg::NSLOT) & 1;
                            ok = mbar_wait(bar_kv_empty + 8 * slot, par ^ 1, abort_flag);
                            if (!ok) break;
                            // test hook (cp_selftest_stall): the tile is never loaded
                            if (P.stall == 8 /* CP_K_BWD_DQ */ && blockIdx.x == 0 && nload == 0) continue;
                            mbar_arrive_expect_tx(bar_kv_full + 8 * slot, Cfg::KTILE);
                            for (int h = 0; h < D / 64; ++h)
                                tma_load_2d(sKV + slot * Cfg::KTILE + h * 16384,
                                            kv == 0 ? (const void*)&tmK : (const void*)&tmV, h * 64,
                                            it.bkv * P.kv_rows + (kpos - (P.kv_base < 0 ? j * n2c : P.kv_base)),
                                            bar_kv_full + 8 * slot);
                        }
                    }
                }
            }
            if (!ok) {
                for (uint32_t n = (nload > Cfg::NSLOT ? nload - Cfg::NSLOT : 0); n < nload; ++n)
                    mbar_wait_drain(bar_kv_full + 8 * (n % Cfg::NSLOT), (n / Cfg::NSLOT) & 1);
            }
        }
      } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the control flow; one elected lane issues each group
        // of tensor-core instructions.  Order per key tile i: S(i) (once the
        // elementwise warps have copied out S(i-1)), dQ += dS(i-1) K(i-1) (dS sits
        // in the dP columns), then dP(i) over them (the tensor pipe runs in order).
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
            constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);   // A tmem, B MN-major
            constexpr uint32_t KT16 = Cfg::KTILE >> 4;
            const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256, tQ = tmem + 384, tdO = tmem + 448;
            const uint64_t dKV = sdesc_sw128(sKV, 16, 1024), dKVmn = sdesc_sw128(sKV, 16384, 1024);
            uint32_t nload = 0, iter = 0, sf_phase = 0, ae_phase = 0;
            uint32_t p_phase[BWD_NSLICE];
            for (int i = 0; i < BWD_NSLICE; ++i) p_phase[i] = 0;
            bool ok = true, acc_busy = false, s_pending = false;
            // dQ += dS K for one finished key tile; dS of slice j (64 keys) sits at dP
            // columns 64j + 16w (keys 64j + 16w .. +15, over the dP columns that warp read)
            auto issue_dq = [&](uint32_t kslot, bool& first) -> bool {
                if (first && acc_busy) {   // every group has stored the previous item's dQ
                    if (!mbar_wait_warp(bar_acc_empty, ae_phase, abort_flag)) return false;
                    ae_phase ^= 1;
                    acc_busy = false;
                }
                const uint64_t bk_mn = dKVmn + kslot * KT16;
                for (int j = 0; j < BWD_NSLICE; ++j) {
                    if (!mbar_wait_warp(bar_p_full + 8 * j, p_phase[j], abort_flag)) return false;
                    p_phase[j] ^= 1;
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4)
                            mma_ts(tdQ, tdP + 64 * j + 16 * w4, bk_mn + (((4 * j + w4) * 2048) >> 4), IDESC_G,
                                   (!first || j > 0 || w4 > 0) ? 1u : 0u);
                    }
                    __syncwarp();
                }
                first = false;
                if (elect_one()) mma_commit(bar_kv_empty + 8 * kslot);
                __syncwarp();
                return true;
            };
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const DqItem it = decode_dq<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                ok = mbar_wait_warp(bar_qt_full, iter & 1, abort_flag);   // Q, dO rows in tensor memory
                if (!ok) break;
                tc_fence_after();
                bool first = true, prev_live = false;
                uint32_t prev_kslot = 0;
                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int ko = tile_orig_of<PD>(P, j, kt, half);
                        if (classify_tile(it.qo, dsf, dsl, ko, P.nc) == TILE_SKIP) continue;
                        const uint32_t kslot = nload % Cfg::NSLOT, kpar = (nload / Cfg::NSLOT) & 1;
                        const uint32_t vslot = (nload + 1) % Cfg::NSLOT, vpar = ((nload + 1) / Cfg::NSLOT) & 1;
                        nload += 2;
                        ok = mbar_wait_warp(bar_kv_full + 8 * kslot, kpar, abort_flag);
                        if (!ok) break;
                        if (s_pending) {   // S of the previous tile is copied out
                            ok = mbar_wait_warp(bar_s_free, sf_phase, abort_flag);
                            if (!ok) break;
                            sf_phase ^= 1;
                        }
                        tc_fence_after();
                        const uint64_t bk = dKV + kslot * KT16, bv = dKV + vslot * KT16;
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ts(tS, tQ + 8 * k, bk + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_st_ready);
                        }
                        __syncwarp();
                        s_pending = true;
                        // the previous tile's products read dS from the dP columns ...
                        if (prev_live && !(ok = issue_dq(prev_kslot, first))) break;
                        // ... before this tile's dP overwrites them
                        ok = mbar_wait_warp(bar_kv_full + 8 * vslot, vpar, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ts(tdP, tdO + 8 * k, bv + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_dp_ready);
                            mma_commit(bar_kv_empty + 8 * vslot);
                        }
                        __syncwarp();
                        prev_live = true;
                        prev_kslot = kslot;
                    }
                }
                if (!ok) break;
                if (elect_one()) mma_commit(bar_qt_empty);   // the item's last S / dP are issued
                __syncwarp();
                if (prev_live) ok = issue_dq(prev_kslot, first);
                if (!ok) break;
                if (elect_one()) {
                    if (!first) mma_commit(bar_acc_full);   // the elementwise groups wait only if they had a tile
                }
                __syncwarp();
                acc_busy = acc_busy || !first;
            }
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            mbar_wait_drain(bar_drain, 0);
        }
      }
    } else {
        regs_inc<104>();
        // ------------------------------------------------------------ elementwise groups (query rows)
        const int wg = warp >> 2;                        // key columns [16wg, 16wg+16) of each slice
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 16 * wg, tdP = tmem + lane_off + 128 + 16 * wg;
        const uint32_t tdQ = tmem + lane_off + 256 + 32 * wg;
        const uint32_t tQ = tmem + lane_off + 384 + 16 * wg, tdO = tmem + lane_off + 448 + 16 * wg;
        // packed dS of slice j goes to dP columns 64j + 8wg
        // packed dS of slice j goes over this warp's own dP columns, already read: 64j + 16wg
        const uint32_t tDs = tmem + lane_off + 128 + 16 * wg;
        uint32_t st_phase = 0, dp_phase = 0, a_phase = 0, iter = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
            const DqItem it = decode_dq<PD>(P, w);
            const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
            const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
            const size_t rowi = static_cast<size_t>(it.bh) * P.q_rows + (it.qpos - P.q_base) + row;
            // this row's Q and dO (bf16 pairs, columns [32wg, 32wg+32)) into tensor memory once the
            // previous item's S / dP have read the old ones
            ok = __all_sync(0xffffffffu, mbar_wait(bar_qt_empty, (iter & 1) ^ 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            if (32 * wg < D) {
                const uint4* qsrc = reinterpret_cast<const uint4*>(P.q + rowi * D + 32 * wg);
                const uint4* osrc = reinterpret_cast<const uint4*>(P.dout + rowi * D + 32 * wg);
                uint32_t qa[16], oa[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 x = __ldg(qsrc + i), y = __ldg(osrc + i);
                    qa[4 * i] = x.x; qa[4 * i + 1] = x.y; qa[4 * i + 2] = x.z; qa[4 * i + 3] = x.w;
                    oa[4 * i] = y.x; oa[4 * i + 1] = y.y; oa[4 * i + 2] = y.z; oa[4 * i + 3] = y.w;
                }
                tmem_st16(tQ, qa);
                tmem_st16(tdO, oa);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_qt_full);
            const float nlse2 = __ldg(P.nlse2 + rowi);
            const float dlt = __ldg(P.delta + rowi);
            const int q_orig = it.qo + row;
            const int ds_q = max(P.docs ? __ldg(P.doc_start + it.qpos + row) : 0, q_orig - P.wm1);
            bool had = false;
            for (int s = P.s0; s < P.s1 && ok; ++s) {
                const int j = __ldg(P.src + it.r * P.cp + s);
                const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                    const int ko = tile_orig_of<PD>(P, j, kt, half);
                    const int cls = classify_tile(it.qo, dsf, dsl, ko, P.nc);
                    if (cls == TILE_SKIP) continue;
                    // ---- S: copy out, release, and form P while dP is still being computed
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_st_ready, st_phase, abort_flag));
                    if (!ok) break;
                    st_phase ^= 1;
                    tc_fence_after();
                    const int lo = ds_q - ko - 16 * wg, hi = q_orig + P.nc - ko - 16 * wg;
                    float sv[32], dp[32];
                    tmem_ld16f(tS, sv);
                    tmem_ld16f(tS + 64, sv + 16);
                    tmem_wait_ld();
                    reg_fence32f(sv);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_s_free);   // the MMA warp may compute the next S
#pragma unroll
                    for (int jj = 0; jj < BWD_NSLICE; ++jj) {
                        if (cls == TILE_FULL)
                            dq_p16<false>(sv + 16 * jj, nlse2, P.scale_log2, 0, 0);
                        else
                            dq_p16<true>(sv + 16 * jj, nlse2, P.scale_log2, lo - 64 * jj, hi - 64 * jj);
                    }
                    // ---- dP: copy out; the packed dS goes over this warp's own columns
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_ready, dp_phase, abort_flag));
                    if (!ok) break;
                    dp_phase ^= 1;
                    tc_fence_after();
                    tmem_ld16f(tdP, dp);
                    tmem_ld16f(tdP + 64, dp + 16);
                    tmem_wait_ld();
                    reg_fence32f(dp);
#pragma unroll
                    for (int jj = 0; jj < BWD_NSLICE; ++jj) {
                        uint32_t dk[8];
                        dq_ds16(sv + 16 * jj, dp + 16 * jj, dlt, dk);
                        tmem_st8(tDs + 64 * jj, dk);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_full + 8 * jj);
                    }
                    had = true;
                }
            }
            if (!ok) break;
            if (had) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full, a_phase, abort_flag));
                if (!ok) break;
                a_phase ^= 1;
                tc_fence_after();
                if (32 * wg < D) {
                    float a[32];
                    tmem_ld32f(tdQ, a);
                    tmem_wait_ld();
                    reg_fence32f(a);
                    if (P.dq32) {   // fp32 dQ, added into the caller's sum (this CTA owns the row)
                        float4* dq = reinterpret_cast<float4*>(P.dq32 + rowi * D + 32 * wg);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float4 x = make_float4(a[4 * i] * P.scale, a[4 * i + 1] * P.scale,
                                                   a[4 * i + 2] * P.scale, a[4 * i + 3] * P.scale);
                            if (P.accumulate) {
                                const float4 u = dq[i];
                                x.x += u.x; x.y += u.y; x.z += u.z; x.w += u.w;
                            }
                            dq[i] = x;
                        }
                    } else {
                    uint4* dq = reinterpret_cast<uint4*>(P.dq + rowi * D + 32 * wg);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dq[i] = make_uint4(pack_bf16(a[8 * i] * P.scale, a[8 * i + 1] * P.scale),
                                           pack_bf16(a[8 * i + 2] * P.scale, a[8 * i + 3] * P.scale),
                                           pack_bf16(a[8 * i + 4] * P.scale, a[8 * i + 5] * P.scale),
                                           pack_bf16(a[8 * i + 6] * P.scale, a[8 * i + 7] * P.scale));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty);
            } else if (32 * wg < D && !P.accumulate) {
                if (P.dq32) {
                    float4* dq = reinterpret_cast<float4*>(P.dq32 + rowi * D + 32 * wg);
                    for (int i = 0; i < 8; ++i) dq[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    uint4* dq = reinterpret_cast<uint4*>(P.dq + rowi * D + 32 * wg);
                    for (int i = 0; i < 4; ++i) dq[i] = make_uint4(0, 0, 0, 0);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        __syncwarp();
        tc_fence_after();
        tmem_relinquish();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace cpattn
