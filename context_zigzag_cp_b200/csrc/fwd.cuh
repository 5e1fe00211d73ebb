// Forward kernel: causal (optionally packed-document, optionally sliding-window)
// attention of every virtual rank's query shard against the K/V shards in the
// plan's visit order.
//
// Work item = (batch*head, a pair of adjacent 128-row query tiles inside one
// zigzag chunk).  Items run GQA group by group; inside a group by descending
// original query position (the longest items start first) with the group's
// query heads fastest, dealt round-robin to one persistent CTA per SM.
//
// Warp roles (384 threads = three warpgroups):
//   warps 0-3  softmax group 0 (query tile 0): one TMEM lane = one query row
//   warps 4-7  softmax group 1 (query tile 1)
//   warp 8     TMA producer: Q tiles, then K and V tiles through a ring of
//              shared-memory slots
//   warp 9     MMA issuer (one elected lane per group of MMAs) + tensor-memory owner
//   warps 10-11 idle
// The block launches with 168 registers per thread; the softmax warpgroups
// raise theirs to 200 and the producer/MMA warpgroup drops to 104
// (2*128*200 + 128*104 = 384*168).
// Tensor memory (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,256+D),
// O1 [384,384+D).  P is written back as bf16 over the first 64 columns of its
// S region and used as the A operand of O += P V straight from tensor memory.
//
// Per KV tile t the MMA warp issues, for each query tile X that the tile
// does not skip:  O_X += P_X(prev) V(prev)  then  S_X = Q_X K_t^T, so the
// tensor core computes S for one query tile while the other group runs its
// softmax (ping-pong between the two groups).
//
// Visit order: for virtual rank r the K/V shards are visited as src[r][s],
// s = 0..cp-1 (all-gather: rank order; ring: (r - s) mod cp).  With
// CP_MERGE_SEPARATE each step is one segment whose partial (O, LSE) is
// written in fp32 and later combined by the merge kernel; with
// CP_MERGE_FUSED the whole visit is one segment and the combine happens in the
// running online-softmax state, step after step, in the same order.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "exp2_poly.cuh"
#include "zigzag.cuh"

namespace cpattn {

struct FwdParams {
    int32_t BH, Hq, Hkv, S, cp, C;  // BH = batch * Hq
    int32_t docs;                   // 1 = packed-document mask
    int32_t wm1;                    // sliding window - 1 (larger than S: no window)
    int32_t nc;                     // last visible key of query q is q + nc: 0 causal, S none
    int32_t fused;                  // 1 = CP_MERGE_FUSED
    int32_t parts_tiled;            // separate merge: partials tile-interleaved (lse_merge_tiled_kernel)
                                    // rather than row-major [parts][rows][D]
    float scale_log2;               // softmax scale * log2(e)
    int32_t n_items, ppc;           // items, query-tile pairs per chunk
    int32_t stall;                  // test hook: 1 = CTA 0 skips its first K/V load
    // Row layouts.  Q / O / LSE (and partials) hold q_rows rows per batch*head whose
    // first row is shard position q_base (S and 0 for the whole sequence; 2C and
    // r*2C for rank r's local shard).  K / V hold kv_rows rows per batch*KV head
    // starting at shard position kv_base (S and 0 gathered); kv_base = -1: they hold
    // only the shard being visited (2C rows: the one shard of a ring step).
    int32_t q_rows, q_base, kv_rows, kv_base;
    int32_t rank;                   // -1: the items of every rank; r: rank r's only
    int32_t s0, s1;                 // visit steps s0 .. s1-1 (partials indexed s - s0)
    // per-document plans: original start of each 128-row shard tile and its inverse
    // ([S/128] each); null for the sequence-level zigzag (closed forms instead)
    const int32_t* tile_orig;
    const int32_t* tile_shard;
    const int32_t* src;             // [cp*cp]
    const int32_t* doc_start;       // [S] shard order
    const __nv_bfloat16* q;         // [BH][q_rows][D] (read directly by the head_dim-256 kernel)
    __nv_bfloat16* o;               // [BH][S][D]  (fused)
    float* lse;                     // [BH][S]     (fused)
    float* o_parts;                 // [cp][BH][S][D] (separate)
    float* lse_parts;               // [cp][BH][S]    (separate)
};

enum : int { TILE_SKIP = 0, TILE_FULL = 1, TILE_PARTIAL = 2 };

// Query tile rows have original positions [qo, qo+127] and first visible keys
// (document start, raised to q - W + 1 under a sliding window) between dsf
// (first row) and dsl (last row); key tile keys [ko, ko+127].  A pair (q, k)
// is admitted when first(q) <= k <= q + nc: nc = 0 is the causal mask, nc = S
// (larger than any k - q) leaves keys unbounded above (no causal mask).
__device__ __forceinline__ int classify_tile(int qo, int dsf, int dsl, int ko, int nc)
{
    if (ko > qo + 127 + nc || ko + 127 < dsf) return TILE_SKIP;
    if (ko + 127 <= qo + nc && ko >= dsl) return TILE_FULL;
    return TILE_PARTIAL;
}

struct FwdItem {
    int bh, bkv, r, p0, ntq;
    int qo[2];   // original start of the item's query tiles
};

// Original start of key tile kt (0 <= kt < 2C/128) of shard j: the first C/128
// tiles are chunk j, the rest chunk 2cp-1-j.  No division: every role calls
// this once per key tile.
__device__ __forceinline__ int key_tile_orig(int j, int kt, int half, int C, int cp)
{
    return kt < half ? j * C + kt * 128 : (2 * cp - 1 - j) * C + (kt - half) * 128;
}

// Items run GQA group by group (a group: one KV head and its g query heads);
// inside a group, 256-row query units by descending original position (the
// longest first) with the group's query heads fastest.  The CTAs in flight then
// stream the K/V tiles of one KV head, which stay in L2.
// The key tiles of shard j (kt < 2C/128: the first C/128 tiles are chunk j,
// the rest chunk 2cp-1-j) that can hold a key in [lo, hi]: kt in [a0, b0) or
// [a1, b1).  Loops visit only these (for (kt = kt_first(r); kt < r.b1;
// kt = kt_next(r, kt))); the tiles outside are skip tiles under every mask, so
// walking them one by one would only cost time (much of it under a sliding
// window).  An empty first range is [0, 0), an empty second one [half, half).
struct KtSpan {
    int a0, b0, a1, b1;
};

__device__ __forceinline__ KtSpan kt_span(int j, int lo, int hi, int half, int C, int cp)
{
    KtSpan r;
    const int c0 = j * C, c1 = (2 * cp - 1 - j) * C;
    r.a0 = max(0, (lo - c0) >> 7);                 // arithmetic shift: floor division by 128
    r.b0 = min(half, ((hi - c0) >> 7) + 1);
    if (r.a0 >= r.b0) r.a0 = r.b0 = 0;
    r.a1 = half + max(0, (lo - c1) >> 7);
    r.b1 = half + min(half, ((hi - c1) >> 7) + 1);
    if (r.a1 >= r.b1) r.a1 = r.b1 = half;
    return r;
}

__device__ __forceinline__ int kt_first(const KtSpan& r) { return r.a0 < r.b0 ? r.a0 : r.a1; }
__device__ __forceinline__ int kt_next(const KtSpan& r, int kt) { return kt + 1 == r.b0 ? r.a1 : kt + 1; }

// The zigzag maps, from the plan's tile tables for per-document plans (PD: tiles
// of a shard are then pieces of many documents) and in closed form otherwise.
// The kernels are compiled once for each, so the sequence path carries no table
// code.  PP is FwdParams or BwdParams.
// Original start of key tile kt (0 <= kt < 2C/128) of shard j.
template <bool PD, class PP>
__device__ __forceinline__ int tile_orig_of(const PP& P, int j, int kt, int half)
{
    if (PD) return __ldg(P.tile_orig + j * 2 * half + kt);
    return key_tile_orig(j, kt, half, P.C, P.cp);
}
// The key tiles of shard j that can hold a key in [lo, hi].  Under a
// per-document plan a shard holds its two chunks of every document in document
// order (chunk j before chunk 2cp-1-j), so the original starts of its tiles
// increase along the shard and the tiles that can hold such a key are one run,
// found by two binary searches of the tile table (both stay inside the shard's
// 2C/128 entries whatever the table holds).
template <bool PD, class PP>
__device__ __forceinline__ KtSpan kv_span(const PP& P, int j, int lo, int hi, int half)
{
    if (PD) {
        const int32_t* t = P.tile_orig + j * 2 * half;
        int a = 0, b = 2 * half;
        while (a < b) {                        // first tile whose last key is >= lo
            const int m = (a + b) >> 1;
            if (__ldg(t + m) + 127 < lo) a = m + 1; else b = m;
        }
        const int first = a;
        b = 2 * half;
        while (a < b) {                        // first tile starting after hi
            const int m = (a + b) >> 1;
            if (__ldg(t + m) <= hi) a = m + 1; else b = m;
        }
        KtSpan r;
        r.a0 = first;
        r.b0 = r.a1 = r.b1 = a;
        return r;
    }
    return kt_span(j, lo, hi, half, P.C, P.cp);
}
// Shard position of the 128-row tile that starts at original position qo.
template <bool PD, class PP>
__device__ __forceinline__ int shard_of_tile(const PP& P, int qo)
{
    if (PD) return __ldg(P.tile_shard + (qo >> 7)) * 128;
    return shard_of_orig(qo, P.C, P.cp);
}
// Original start of the 128-row tile at shard position qpos.
template <bool PD, class PP>
__device__ __forceinline__ int orig_of_tile(const PP& P, int qpos)
{
    if (PD) return __ldg(P.tile_orig + (qpos >> 7));
    return orig_of_shard(qpos, P.C, P.cp);
}

// Chunks an item list covers: all 2cp, or rank r's two (its tail chunk first).
__device__ __forceinline__ int fwd_nchunks(const FwdParams& P) { return P.rank < 0 ? 2 * P.cp : 2; }

template <bool PD>
__device__ __forceinline__ FwdItem decode_item(const FwdParams& P, int w)
{
    FwdItem it;
    const int g = P.Hq / P.Hkv;
    if (PD) {
        // per-document plans: 256-row units of shard positions (the rank's, or all),
        // by descending shard position; each unit holds two whole tiles (2C is a
        // multiple of 256) whose original starts come from the plan
        const int nunits = (P.rank < 0 ? P.S : 2 * P.C) / 256;
        const int per_group_d = g * nunits;
        it.bkv = w / per_group_d;
        const int rem = w - it.bkv * per_group_d;
        const int t = rem / g, hq = rem - t * g;
        const int b = it.bkv / P.Hkv, hk = it.bkv - b * P.Hkv;
        it.bh = b * P.Hq + hk * g + hq;
        it.p0 = (P.rank < 0 ? 0 : P.rank * 2 * P.C) + (nunits - 1 - t) * 256;
        it.r = it.p0 / (2 * P.C);
        it.qo[0] = __ldg(P.tile_orig + (it.p0 >> 7));
        it.qo[1] = __ldg(P.tile_orig + (it.p0 >> 7) + 1);
        it.ntq = 2;
        return it;
    }
    const int per_group = g * fwd_nchunks(P) * P.ppc;
    it.bkv = w / per_group;
    const int rem = w - it.bkv * per_group;
    const int t = rem / g, hq = rem - t * g;
    const int b = it.bkv / P.Hkv, hk = it.bkv - b * P.Hkv;
    it.bh = b * P.Hq + hk * g + hq;
    const int u = P.ppc - 1 - t % P.ppc;
    const int ci = t / P.ppc;                // original chunk, descending
    const int c = P.rank < 0 ? 2 * P.cp - 1 - ci : (ci == 0 ? 2 * P.cp - 1 - P.rank : P.rank);
    int half;
    if (c < P.cp) { it.r = c; half = 0; } else { it.r = 2 * P.cp - 1 - c; half = 1; }
    it.p0 = it.r * 2 * P.C + half * P.C + u * 256;
    it.qo[0] = c * P.C + u * 256;
    it.qo[1] = it.qo[0] + 128;
    it.ntq = (u * 256 + 256 <= P.C) ? 2 : 1;
    return it;
}

// K/V ring slots of the forward at head_dim 128: 5 (Q tiles 64 KB + ring 160 KB
// fit the 227 KB a CTA may use); measured 3.5 % faster than 4 at gqa32k.
#ifndef CP_FWD_NSLOT128
#define CP_FWD_NSLOT128 5
#endif

template <int D>
struct FwdCfg {
    static constexpr int TILE_BYTES = 128 * D * 2;      // one 128-row bf16 tile
    static constexpr int NSLOT = (D == 128) ? CP_FWD_NSLOT128 : 8;   // K/V ring slots
    static constexpr int Q_OFF = 0;                     // Q0, Q1
    static constexpr int KV_OFF = 2 * TILE_BYTES;
    static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
    // barriers: q_full, q_empty, s_full[2], p_full[2], o_full[2], kv_full[NSLOT], kv_empty[NSLOT], drain
    static constexpr int NBAR = 9 + 2 * NSLOT;
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64 + 1024;  // + alignment slack
    static constexpr int THREADS = 384;
};

struct TileIter {
    // per-item geometry shared by every role
    int qo[2], dsf[2], dsl[2];
};

// Original start of each query tile of an item and the range of its rows'
// first visible key, max(document start, q - wm1), over the tile (first row,
// last row); the second tile exists only when it.ntq == 2 (no read past the
// item's rows).
__device__ __forceinline__ TileIter load_tile_iter(const FwdParams& P, const FwdItem& it)
{
    TileIter ti;
    for (int x = 0; x < 2; ++x) {
        ti.qo[x] = it.qo[x];
        ti.dsf[x] = 0;
        ti.dsl[x] = 0;
        if (P.docs && x < it.ntq) {
            const int pr = it.p0 + 128 * x;
            ti.dsf[x] = __ldg(P.doc_start + pr);
            ti.dsl[x] = __ldg(P.doc_start + pr + 127);
        }
        ti.dsf[x] = max(ti.dsf[x], ti.qo[x] - P.wm1);
        ti.dsl[x] = max(ti.dsl[x], ti.qo[x] + 127 - P.wm1);
    }
    return ti;
}

// Of every four column pairs of an unmasked tile, this many take 2^x from the
// software exp2 on the FMA pipe (exp2_poly.cuh), the rest from ex2.approx.
// Measured on B200 (gqa32k, long128k): 0 is fastest; 1 of 4 costs 1-2 %, 2 of
// 4 costs 3-5 %, so the special-function pipe does not set the forward's pace.
#ifndef CP_FWD_POLY_PAIRS
#define CP_FWD_POLY_PAIRS 0
#endif

// Exponentials of one query row's 128 scores (log2 domain, reference max msub),
// packed to bf16 pairs and stored over the first 64 columns of the row's S
// region; returns the fp32 row sum.  NSOFT of every four pairs of columns use
// the software exp2 on the FMA pipe (only for unmasked tiles, whose arguments
// are finite), the rest the hardware ex2.
template <int NSOFT>
__device__ __forceinline__ float exp_pack_store(const float* sf, float scale_log2, float msub,
                                                uint32_t tS)
{
    const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
    const uint64_t nm = f2_pack(-msub, -msub);
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint64_t x2 = f2_fma(f2_pack(sf[64 * h + 2 * i], sf[64 * h + 2 * i + 1]), sl2, nm);
            uint64_t p2;
            if ((i & 3) >= 4 - NSOFT) {
                p2 = exp2_poly2(x2);
            } else {
                float a, b;
                f2_unpack(x2, a, b);
                p2 = f2_pack(ex2_approx(a), ex2_approx(b));
            }
            acc[i & 3] = f2_add(acc[i & 3], p2);
            float a, b;
            f2_unpack(p2, a, b);
            pk[i] = pack_bf16(a, b);
        }
        tmem_st32(tS + 32 * h, pk);
    }
    const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    float a, b;
    f2_unpack(t, a, b);
    return a + b;
}

template <int D, bool PD>
__global__ void __launch_bounds__(384, 1)
cp_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const FwdParams P)
{
    using Cfg = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ0 = sbase + Cfg::Q_OFF, sKV = sbase + Cfg::KV_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_q_full = bars, bar_q_empty = bars + 8;
    const uint32_t bar_s_full = bars + 16, bar_p_full = bars + 32, bar_o_full = bars + 48;
    const uint32_t bar_kv_full = bars + 64, bar_kv_empty = bars + 64 + 8 * Cfg::NSLOT;
    const uint32_t bar_drain = bars + 64 + 16 * Cfg::NSLOT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8 + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n2c = 2 * P.C;
    const int half = P.C / 128;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_s_full + 8 * x, 1);
            mbar_init(bar_p_full + 8 * x, 4);
            mbar_init(bar_o_full + 8 * x, 1);
        }
        for (int i = 0; i < Cfg::NSLOT; ++i) {
            mbar_init(bar_kv_full + 8 * i, 1);
            mbar_init(bar_kv_empty + 8 * i, 1);
        }
        mbar_init(bar_drain, 1);
        fence_barrier_init();
    }
    if (warp == 9) tmem_alloc(smem_u32(tmem_slot), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp >= 8) {
      regs_dec<104>();
      if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t nload = 0, iter = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const FwdItem it = decode_item<PD>(P, w);
                const TileIter ti = load_tile_iter(P, it);
                ok = mbar_wait(bar_q_empty, (iter & 1) ^ 1, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_q_full, it.ntq * Cfg::TILE_BYTES);
                for (int x = 0; x < it.ntq; ++x)
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_2d(sQ0 + x * Cfg::TILE_BYTES + h * 16384, &tmQ, h * 64,
                                    it.bh * P.q_rows + (it.p0 - P.q_base) + 128 * x, bar_q_full);
                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, ti.dsf[0], (it.ntq == 2 ? ti.qo[1] : ti.qo[0]) + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int kpos = j * n2c + kt * 128;
                        const int ko = tile_orig_of<PD>(P, j, kt, half);
                        const bool v0 = classify_tile(ti.qo[0], ti.dsf[0], ti.dsl[0], ko, P.nc) != TILE_SKIP;
                        const bool v1 = it.ntq == 2 &&
                                        classify_tile(ti.qo[1], ti.dsf[1], ti.dsl[1], ko, P.nc) != TILE_SKIP;
                        if (!v0 && !v1) continue;
                        for (int kv = 0; kv < 2 && ok; ++kv, ++nload) {
                            const uint32_t slot = nload % Cfg::NSLOT;
                            const uint32_t par = (nload / Cfg::NSLOT) & 1;
                            ok = mbar_wait(bar_kv_empty + 8 * slot, par ^ 1, abort_flag);
                            if (!ok) break;
                            // test hook (cp_selftest_stall): the tile is never loaded, so the
                            // MMA warp's bounded wait on it runs out and the CTA tears down
                            if (P.stall && blockIdx.x == 0 && nload == 0) continue;
                            mbar_arrive_expect_tx(bar_kv_full + 8 * slot, Cfg::TILE_BYTES);
                            for (int h = 0; h < D / 64; ++h)
                                tma_load_2d(sKV + slot * Cfg::TILE_BYTES + h * 16384,
                                            kv == 0 ? (const void*)&tmK : (const void*)&tmV, h * 64,
                                            it.bkv * P.kv_rows + (kpos - (P.kv_base < 0 ? j * n2c : P.kv_base)),
                                            bar_kv_full + 8 * slot);
                        }
                    }
                }
            }
            if (!ok) {
                // abort path: let the copies already issued land before the CTA exits
                for (uint32_t n = (nload > Cfg::NSLOT ? nload - Cfg::NSLOT : 0); n < nload; ++n)
                    mbar_wait_drain(bar_kv_full + 8 * (n % Cfg::NSLOT), (n / Cfg::NSLOT) & 1);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the control flow; one elected lane issues each group
        // of tensor-core instructions (cheaper than a single diverged lane).
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);
            constexpr uint32_t TILE16 = Cfg::TILE_BYTES >> 4;   // tile stride in descriptor units
            // descriptors of Q tile 0 and KV slot 0; the others are constant offsets
            const uint64_t dq0 = sdesc_sw128(sQ0, 16, 1024);
            const uint64_t dk0 = sdesc_sw128(sKV, 16, 1024);
            const uint64_t dv0 = sdesc_sw128(sKV, 16384, 1024);
            const uint32_t tS0 = tmem, tO0 = tmem + 256;
            uint32_t ring_slot = 0, ring_par = 0, iter = 0;
            uint32_t p_phase0 = 0, p_phase1 = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const FwdItem it = decode_item<PD>(P, w);
                const TileIter ti = load_tile_iter(P, it);
                // number of loaded tiles of this item: Q is released to the producer
                // right after the last S = Q K^T, before the item's final PVs
                int n_tiles = 0;
                for (int s = P.s0; s < P.s1; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, ti.dsf[0], (it.ntq == 2 ? ti.qo[1] : ti.qo[0]) + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1; kt = kt_next(ks, kt)) {
                        const int ko = tile_orig_of<PD>(P, j, kt, half);
                        if (classify_tile(ti.qo[0], ti.dsf[0], ti.dsl[0], ko, P.nc) != TILE_SKIP ||
                            (it.ntq == 2 && classify_tile(ti.qo[1], ti.dsf[1], ti.dsl[1], ko, P.nc) != TILE_SKIP))
                            ++n_tiles;
                    }
                }
                int tiles_done = 0;
                ok = mbar_wait_warp(bar_q_full, iter & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool pend0 = false, pend1 = false;       // a PV of the previous tile is due
                bool first0 = true, first1 = true;       // next PV starts the accumulator
                bool had0 = false, had1 = false;         // query tile had a tile in this segment
                bool pv_live = false;                    // the previous tile's V slot is held
                uint32_t pv_slot = 0, pv_par = 0;

                // O_x += P_x V(previous tile), once softmax group x has written P_x
                auto issue_pv = [&](int x, uint32_t& pph, bool& first) -> bool {
                    if (!mbar_wait_warp(bar_p_full + 8 * x, pph, abort_flag)) return false;
                    pph ^= 1;
                    if (!mbar_wait_warp(bar_kv_full + 8 * pv_slot, pv_par, abort_flag)) return false;
                    tc_fence_after();
                    const uint64_t bv = dv0 + pv_slot * TILE16;
                    const uint32_t ts = tS0 + 128 * x, to = tO0 + 128 * x;
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(to, ts + 8 * k, bv + k * (2048 >> 4), IDESC_PV, (!first || k > 0) ? 1u : 0u);
                    }
                    __syncwarp();
                    first = false;
                    return true;
                };
                auto issue_s = [&](int x, uint32_t kslot) {
                    const uint64_t aq = dq0 + x * TILE16, bk = dk0 + kslot * TILE16;
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                            mma_ss(tS0 + 128 * x, aq + off, bk + off, IDESC_S, k > 0 ? 1u : 0u);
                        }
                        mma_commit(bar_s_full + 8 * x);
                    }
                    __syncwarp();
                };

                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, ti.dsf[0], (it.ntq == 2 ? ti.qo[1] : ti.qo[0]) + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int ko = tile_orig_of<PD>(P, j, kt, half);
                        const bool v0 = classify_tile(ti.qo[0], ti.dsf[0], ti.dsl[0], ko, P.nc) != TILE_SKIP;
                        const bool v1 = it.ntq == 2 && classify_tile(ti.qo[1], ti.dsf[1], ti.dsl[1], ko, P.nc) != TILE_SKIP;
                        if (!v0 && !v1) continue;
                        const uint32_t kslot = ring_slot, kpar = ring_par;
                        if (++ring_slot == Cfg::NSLOT) { ring_slot = 0; ring_par ^= 1; }
                        const uint32_t vslot = ring_slot, vpar = ring_par;
                        if (++ring_slot == Cfg::NSLOT) { ring_slot = 0; ring_par ^= 1; }
                        ok = mbar_wait_warp(bar_kv_full + 8 * kslot, kpar, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        // A pending PV never outlives one tile: it is issued at the next loaded
                        // tile whether or not that tile is valid for its query tile, so a V slot
                        // is held for at most one tile and the ring cannot stall.
                        if (pend0) { ok = issue_pv(0, p_phase0, first0); pend0 = false; }
                        if (ok && v0) { issue_s(0, kslot); pend0 = true; had0 = true; }
                        if (ok && pend1) { ok = issue_pv(1, p_phase1, first1); pend1 = false; }
                        if (ok && v1) { issue_s(1, kslot); pend1 = true; had1 = true; }
                        if (!ok) break;
                        if (elect_one()) {
                            if (pv_live) mma_commit(bar_kv_empty + 8 * pv_slot);   // every PV on it issued
                            mma_commit(bar_kv_empty + 8 * kslot);
                        }
                        __syncwarp();
                        pv_live = true;
                        pv_slot = vslot;
                        pv_par = vpar;
                        if (++tiles_done == n_tiles) { if (elect_one()) mma_commit(bar_q_empty); __syncwarp(); }
                    }
                    // end of a segment: every step (separate) or the whole visit (fused)
                    if (ok && (!P.fused || s == P.s1 - 1)) {
                        if (pend0) { ok = issue_pv(0, p_phase0, first0); pend0 = false; }
                        if (ok && pend1) { ok = issue_pv(1, p_phase1, first1); pend1 = false; }
                        if (ok && elect_one()) {
                            if (pv_live) mma_commit(bar_kv_empty + 8 * pv_slot);
                            // each softmax group waits for this whenever it had a tile in the
                            // segment, even if its last PV was issued at an earlier tile
                            if (had0) mma_commit(bar_o_full);
                            if (had1) mma_commit(bar_o_full + 8);
                        }
                        __syncwarp();
                        pv_live = false;
                        first0 = first1 = true;
                        had0 = had1 = false;
                    }
                }
                if (ok && n_tiles == 0) { if (elect_one()) mma_commit(bar_q_empty); __syncwarp(); }
            }
            // drain: every MMA and commit issued above has completed
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            mbar_wait_drain(bar_drain, 0);
        }
      }
    } else {
        regs_inc<200>();
        // ------------------------------------------------------------ softmax groups
        const int X = warp >> 2;                 // query tile handled by this group
        const int row = (warp & 3) * 32 + lane;  // TMEM lane == query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128 * X;
        const uint32_t tO = tmem + lane_off + 256 + 128 * X;
        uint32_t s_phase = 0, o_phase = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x) {
            const FwdItem it = decode_item<PD>(P, w);
            if (X >= it.ntq) continue;
            const TileIter ti = load_tile_iter(P, it);
            const int prow = it.p0 + 128 * X + row;      // shard position of my row
            const int q_orig = ti.qo[X] + row;
            const int ds_row = max(P.docs ? __ldg(P.doc_start + prow) : 0, q_orig - P.wm1);
            float m_used = -INFINITY, l_sum = 0.f;
            bool first = true, had = false;
            for (int s = P.s0; s < P.s1 && ok; ++s) {
                const int j = __ldg(P.src + it.r * P.cp + s);
                const KtSpan ks = kv_span<PD>(P, j, ti.dsf[X], ti.qo[X] + 127 + P.nc, half);
                for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                    const int ko = tile_orig_of<PD>(P, j, kt, half);
                    const int cls = classify_tile(ti.qo[X], ti.dsf[X], ti.dsl[X], ko, P.nc);
                    if (cls == TILE_SKIP) continue;
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full + 8 * X, s_phase, abort_flag));
                    if (!ok) break;
                    s_phase ^= 1;
                    tc_fence_after();
                    float sf[128];
                    tmem_ld32f(tS + 0, sf + 0);
                    tmem_ld32f(tS + 32, sf + 32);
                    tmem_ld32f(tS + 64, sf + 64);
                    tmem_ld32f(tS + 96, sf + 96);
                    tmem_wait_ld();
                    reg_fence32f(sf + 0);
                    reg_fence32f(sf + 32);
                    reg_fence32f(sf + 64);
                    reg_fence32f(sf + 96);
                    if (cls == TILE_PARTIAL) {
                        const int lo = ds_row - ko, hi = q_orig + P.nc - ko;
#pragma unroll
                        for (int c = 0; c < 128; ++c)
                            if (c < lo || c > hi) sf[c] = -INFINITY;
                    }
                    float mx4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(sf[i], sf[i + 4]);
#pragma unroll
                    for (int c = 8; c < 128; c += 8)
#pragma unroll
                        for (int i = 0; i < 4; ++i) mx4[i] = fmax3(mx4[i], sf[c + i], sf[c + 4 + i]);
                    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    const float m_tile = mx * P.scale_log2;
                    // lazy rescale: keep the reference max unless it is exceeded by more
                    // than 8 (a factor 256 in the exponentials), or is still -inf
                    const bool need = m_tile > m_used + 8.0f;
                    float alpha = 1.f;
                    if (need) {
                        alpha = ex2_approx(m_used - m_tile);   // 0 when m_used = -inf
                        m_used = m_tile;
                    }
                    if (!first && __any_sync(0xffffffffu, need)) {
                        // O *= alpha for this row (the PV of the previous tile is complete)
#pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 16) {
                            float of[16];
                            tmem_ld16f(tO + c0, of);
                            tmem_wait_ld();
                            reg_fence16f(of);
#pragma unroll
                            for (int i = 0; i < 16; ++i) of[i] *= alpha;
                            tmem_st16f(tO + c0, of);
                        }
                    }
                    const float msub = (m_used == -INFINITY) ? 0.f : m_used;
                    const float rs = cls == TILE_FULL
                                         ? exp_pack_store<CP_FWD_POLY_PAIRS>(sf, P.scale_log2, msub, tS)
                                         : exp_pack_store<0>(sf, P.scale_log2, msub, tS);
                    l_sum = l_sum * alpha + rs;
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_p_full + 8 * X);
                    first = false;
                    had = true;
                }
                if (!ok) break;
                if (!P.fused || s == P.s1 - 1) {
                    // ---- epilogue of the segment
                    const size_t rowi = static_cast<size_t>(it.bh) * P.q_rows + (prow - P.q_base);
                    if (had) {
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_full + 8 * X, o_phase, abort_flag));
                        if (!ok) break;
                        o_phase ^= 1;
                        tc_fence_after();
                        const bool empty = !(l_sum > 0.f);
                        const float inv_l = empty ? 0.f : 1.f / l_sum;
                        const float lse_v = empty ? -INFINITY
                                                  : (m_used + lg2_approx(l_sum)) * 0.69314718055994531f;
#pragma unroll
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            float of[32];
                            tmem_ld32f(tO + c0, of);
                            tmem_wait_ld();
                            reg_fence32f(of);
                            uint32_t orr[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(of[i]);
                            if (P.fused) {
                                uint4* dst = reinterpret_cast<uint4*>(P.o + rowi * D + c0);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    uint4 u;
                                    u.x = pack_bf16(__uint_as_float(orr[8 * i + 0]) * inv_l, __uint_as_float(orr[8 * i + 1]) * inv_l);
                                    u.y = pack_bf16(__uint_as_float(orr[8 * i + 2]) * inv_l, __uint_as_float(orr[8 * i + 3]) * inv_l);
                                    u.z = pack_bf16(__uint_as_float(orr[8 * i + 4]) * inv_l, __uint_as_float(orr[8 * i + 5]) * inv_l);
                                    u.w = pack_bf16(__uint_as_float(orr[8 * i + 6]) * inv_l, __uint_as_float(orr[8 * i + 7]) * inv_l);
                                    dst[i] = u;
                                }
                            } else {
                                const size_t prow_all = static_cast<size_t>(s - P.s0) * P.BH * P.q_rows + rowi;
                                // tile-interleaved: the warp's 32 rows store 512 contiguous bytes
                                float4* dst = P.parts_tiled
                                    ? reinterpret_cast<float4*>(P.o_parts) + ((prow_all >> 7) * (D / 4) + c0 / 4) * 128 + (prow_all & 127)
                                    : reinterpret_cast<float4*>(P.o_parts + prow_all * D + c0);
                                const size_t step = P.parts_tiled ? 128 : 1;
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    dst[i * step] = make_float4(__uint_as_float(orr[4 * i + 0]) * inv_l,
                                                                __uint_as_float(orr[4 * i + 1]) * inv_l,
                                                                __uint_as_float(orr[4 * i + 2]) * inv_l,
                                                                __uint_as_float(orr[4 * i + 3]) * inv_l);
                            }
                        }
                        if (P.fused) P.lse[rowi] = lse_v;
                        else P.lse_parts[static_cast<size_t>(s - P.s0) * P.BH * P.q_rows + rowi] = lse_v;
                    } else if (!P.fused) {
                        P.lse_parts[static_cast<size_t>(s - P.s0) * P.BH * P.q_rows + rowi] = -INFINITY;
                    } else {
                        // no admitted key anywhere (cannot happen for a valid mask): (0, -inf)
                        uint4* dst = reinterpret_cast<uint4*>(P.o + rowi * D);
                        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
                        P.lse[rowi] = -INFINITY;
                    }
                    m_used = -INFINITY;
                    l_sum = 0.f;
                    first = true;
                    had = false;
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_relinquish();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace cpattn
