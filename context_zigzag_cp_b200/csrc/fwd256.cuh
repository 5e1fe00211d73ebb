// Forward at head_dim 256: the same computation as cp_fwd_kernel (per-rank,
// per-step causal / document / window / unmasked attention against the K/V
// shards in visit order, merged by log-sum-exp separately or in the running
// state), laid out for D = 256.
//
// The head_dim-128 layout (two query tiles per CTA, each with S and O in tensor
// memory) needs 2 x (128 + 256) columns at D = 256, more than the 512 there
// are.  Here a CTA works on one 128-row query tile at a time:
//   tensor memory  [0, 64), [64, 128)  S of alternate 64-key tiles (P written
//                                      back over the first 32 columns as bf16
//                                      pairs, the A operand of P V)
//                  [128, 256)          the tile's Q rows as bf16 pairs (the A
//                                      operand of S = Q K^T), written by the
//                                      softmax warps once per item
//                  [256, 512)          the O accumulator
//   shared memory  a 7-slot ring of 64-row K / V tiles (32 KB each, TMA,
//                  128-byte swizzle); no Q tile: with Q in tensor memory the
//                  shared-memory port carries only the K/V copies and the
//                  B operands
// While the softmax warps turn S of key tile k into P, the tensor core computes
// S of tile k+1 and P V of tile k-1.  Warps 0-3: softmax (thread = query row),
// warp 4: TMA producer, warp 5: MMA issue (one elected lane) and TMEM owner.
#pragma once
#include "fwd.cuh"

namespace cpattn {

struct Fwd256Cfg {
    static constexpr int D = 256;
    static constexpr int KT = 64;                       // keys per K/V tile
    static constexpr int TILE_BYTES = KT * D * 2;       // 32 KB: four 8 KB swizzled boxes
    static constexpr int BOX_BYTES = KT * 128;          // 64 columns x 64 rows
    static constexpr int NSLOT = 7;
    static constexpr int KV_OFF = 0;
    static constexpr int BAR_OFF = NSLOT * TILE_BYTES;
    // qt_full, qt_empty, s_full[2], p_full[2], o_done, kv_full[NSLOT], kv_empty[NSLOT], drain
    static constexpr int NBAR = 8 + 2 * NSLOT;
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64 + 1024;  // + alignment slack
    static constexpr int THREADS = 192;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// A 64-key tile [ko, ko+63] against the query tile [qo, qo+127] (as
// classify_tile, for 64 keys).
__device__ __forceinline__ int classify_tile64(int qo, int dsf, int dsl, int ko, int nc)
{
    if (ko > qo + 127 + nc || ko + 63 < dsf) return TILE_SKIP;
    if (ko + 63 <= qo + nc && ko >= dsl) return TILE_FULL;
    return TILE_PARTIAL;
}

// One 128-row query tile of one query head.
struct Q1Item {
    int bkv, bh, r, qpos, qo;
};

// Items run GQA group by group; inside a group, query tiles by descending
// original position (the longest first) with the group's query heads fastest.
// Whole sequence (rank < 0): every tile; rank r: its 2C/128 tiles.
template <bool PD>
__device__ __forceinline__ Q1Item decode_q1(const FwdParams& P, int w)
{
    Q1Item it;
    const int g = P.Hq / P.Hkv;
    const int ntiles = P.q_rows / 128;
    const int per_group = g * ntiles;
    it.bkv = w / per_group;
    const int rem = w - it.bkv * per_group;
    const int t = rem / g, hq = rem - t * g;
    const int b = it.bkv / P.Hkv, hk = it.bkv - b * P.Hkv;
    it.bh = b * P.Hq + hk * g + hq;
    if (P.rank < 0) {
        it.qo = (ntiles - 1 - t) * 128;
        it.qpos = shard_of_tile<PD>(P, it.qo);
    } else if (PD) {
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

// Exponentials of one query row's 64 scores (log2 domain, reference max msub),
// packed to bf16 pairs in pk; returns the fp32 row sum.
__device__ __forceinline__ float exp_pack64(const float* sf, float scale_log2, float msub,
                                            uint32_t (&pk)[32])
{
    const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
    const uint64_t nm = f2_pack(-msub, -msub);
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const uint64_t x2 = f2_fma(f2_pack(sf[2 * i], sf[2 * i + 1]), sl2, nm);
        float a, b;
        f2_unpack(x2, a, b);
        const uint64_t p2 = f2_pack(ex2_approx(a), ex2_approx(b));
        acc[i & 3] = f2_add(acc[i & 3], p2);
        f2_unpack(p2, a, b);
        pk[i] = pack_bf16(a, b);
    }
    const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    float a, b;
    f2_unpack(t, a, b);
    return a + b;
}

template <bool PD>
__global__ void __launch_bounds__(192, 1)
cp_fwd256_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const FwdParams P)
{
    using Cfg = Fwd256Cfg;
    constexpr int D = Cfg::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sKV = sbase + Cfg::KV_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_qt_full = bars, bar_qt_empty = bars + 8;
    const uint32_t bar_s_full = bars + 16, bar_p_full = bars + 32, bar_o_done = bars + 48;
    const uint32_t bar_kv_full = bars + 56, bar_kv_empty = bars + 56 + 8 * Cfg::NSLOT;
    const uint32_t bar_drain = bars + 56 + 16 * Cfg::NSLOT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8 + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n2c = 2 * P.C;
    const int half = P.C / 128;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar_qt_full, 4);
        mbar_init(bar_qt_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_s_full + 8 * b, 1);
            mbar_init(bar_p_full + 8 * b, 4);
        }
        mbar_init(bar_o_done, 1);
        for (int i = 0; i < Cfg::NSLOT; ++i) {
            mbar_init(bar_kv_full + 8 * i, 1);
            mbar_init(bar_kv_empty + 8 * i, 1);
        }
        mbar_init(bar_drain, 1);
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(smem_u32(tmem_slot), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t nload = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x) {
                const Q1Item it = decode_q1<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                        for (int hh = 0; hh < 2 && ok; ++hh) {
                            if (classify_tile64(it.qo, dsf, dsl, ko128 + 64 * hh, P.nc) == TILE_SKIP) continue;
                            const int kpos = j * n2c + kt * 128 + 64 * hh;
                            const int kvrow = it.bkv * P.kv_rows + (kpos - (P.kv_base < 0 ? j * n2c : P.kv_base));
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
                                    tma_load_2d(sKV + slot * Cfg::TILE_BYTES + h * Cfg::BOX_BYTES,
                                                kv == 0 ? (const void*)&tmK : (const void*)&tmV, h * 64,
                                                kvrow, bar_kv_full + 8 * slot);
                            }
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
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, Cfg::KT, false, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);
            constexpr uint32_t TILE16 = Cfg::TILE_BYTES >> 4;
            const uint64_t dk0 = sdesc_sw128(sKV, 16, 1024);                 // K-major K tile
            const uint64_t dv0 = sdesc_sw128(sKV, Cfg::BOX_BYTES, 1024);      // MN-major V tile
            const uint32_t tQ = tmem + 128, tO = tmem + 256;
            uint32_t ring_slot = 0, ring_par = 0, iter = 0, sb = 0;
            uint32_t p_phase = 0;            // bit b: parity of the next wait on p_full[b]
            bool ok = true;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const Q1Item it = decode_q1<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                // loaded tiles of this item: Q's columns are released after the last S
                int n_tiles = 0;
                for (int s = P.s0; s < P.s1; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1; kt = kt_next(ks, kt)) {
                        const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                        for (int hh = 0; hh < 2; ++hh)
                            if (classify_tile64(it.qo, dsf, dsl, ko128 + 64 * hh, P.nc) != TILE_SKIP) ++n_tiles;
                    }
                }
                int tiles_done = 0;
                ok = mbar_wait_warp(bar_qt_full, iter & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool pend = false, first = true;
                uint32_t pv_slot = 0, pv_par = 0, pv_buf = 0;

                // O (+)= P V of the pending tile, once the softmax warps have written its P
                auto issue_pv = [&]() -> bool {
                    if (!mbar_wait_warp(bar_p_full + 8 * pv_buf, (p_phase >> pv_buf) & 1u, abort_flag)) return false;
                    p_phase ^= 1u << pv_buf;
                    if (!mbar_wait_warp(bar_kv_full + 8 * pv_slot, pv_par, abort_flag)) return false;
                    tc_fence_after();
                    if (elect_one()) {
                        const uint64_t bv = dv0 + pv_slot * TILE16;
#pragma unroll
                        for (int k = 0; k < Cfg::KT / 16; ++k)
                            mma_ts(tO, tmem + 64 * pv_buf + 8 * k, bv + k * (2048 >> 4), IDESC_PV,
                                   (!first || k > 0) ? 1u : 0u);
                        mma_commit(bar_o_done);
                        mma_commit(bar_kv_empty + 8 * pv_slot);
                    }
                    __syncwarp();
                    first = false;
                    return true;
                };

                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                        for (int hh = 0; hh < 2 && ok; ++hh) {
                            if (classify_tile64(it.qo, dsf, dsl, ko128 + 64 * hh, P.nc) == TILE_SKIP) continue;
                            const uint32_t kslot = ring_slot, kpar = ring_par;
                            if (++ring_slot == Cfg::NSLOT) { ring_slot = 0; ring_par ^= 1; }
                            const uint32_t vslot = ring_slot, vpar = ring_par;
                            if (++ring_slot == Cfg::NSLOT) { ring_slot = 0; ring_par ^= 1; }
                            ok = mbar_wait_warp(bar_kv_full + 8 * kslot, kpar, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                            // S = Q K^T into buffer sb; its P buffer was read by a P V issued
                            // before this (the tensor core runs them in order)
                            if (elect_one()) {
                                const uint64_t bk = dk0 + kslot * TILE16;
#pragma unroll
                                for (int k = 0; k < D / 16; ++k) {
                                    const uint32_t off = ((k / 4) * Cfg::BOX_BYTES + (k % 4) * 32) >> 4;
                                    mma_ts(tmem + 64 * sb, tQ + 8 * k, bk + off, IDESC_S, k > 0 ? 1u : 0u);
                                }
                                mma_commit(bar_s_full + 8 * sb);
                                mma_commit(bar_kv_empty + 8 * kslot);
                            }
                            __syncwarp();
                            if (++tiles_done == n_tiles) { if (elect_one()) mma_commit(bar_qt_empty); __syncwarp(); }
                            if (pend) { ok = issue_pv(); pend = false; }
                            if (!ok) break;
                            pend = true;
                            pv_slot = vslot;
                            pv_par = vpar;
                            pv_buf = sb;
                            sb ^= 1;
                        }
                    }
                    // end of a segment: every step (separate) or the whole visit (fused)
                    if (ok && (!P.fused || s == P.s1 - 1)) {
                        if (pend) { ok = issue_pv(); pend = false; }
                        first = true;
                    }
                }
                if (ok && n_tiles == 0) { if (elect_one()) mma_commit(bar_qt_empty); __syncwarp(); }
            }
            // drain: every MMA and commit issued above has completed
            if (elect_one()) mma_commit(bar_drain);
            __syncwarp();
            mbar_wait_drain(bar_drain, 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax warps
        const int row = warp * 32 + lane;                       // TMEM lane == query row
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tQ = tmem + lane_off + 128, tO = tmem + lane_off + 256;
        uint32_t s_phase = 0, o_phase = 0, sb = 0, iter = 0;   // s_phase bit b: s_full[b]
        bool ok = true;
        for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
            const Q1Item it = decode_q1<PD>(P, w);
            const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
            const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
            const size_t rowi = static_cast<size_t>(it.bh) * P.q_rows + (it.qpos - P.q_base) + row;
            // this row's Q (bf16 pairs) into tensor memory once the previous item's
            // S products have read the old one
            ok = __all_sync(0xffffffffu, mbar_wait(bar_qt_empty, (iter & 1) ^ 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            {
                const uint4* qsrc = reinterpret_cast<const uint4*>(P.q + rowi * D);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t qa[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint4 x = __ldg(qsrc + 8 * c + i);
                        qa[4 * i] = x.x; qa[4 * i + 1] = x.y; qa[4 * i + 2] = x.z; qa[4 * i + 3] = x.w;
                    }
                    tmem_st32(tQ + 32 * c, qa);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_qt_full);
            const int prow = it.qpos + row;                     // shard position of my row
            const int q_orig = it.qo + row;
            const int ds_row = max(P.docs ? __ldg(P.doc_start + prow) : 0, q_orig - P.wm1);
            float m_used = -INFINITY, l_sum = 0.f;
            bool first = true, had = false;
            for (int s = P.s0; s < P.s1 && ok; ++s) {
                const int j = __ldg(P.src + it.r * P.cp + s);
                const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                    const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                    for (int hh = 0; hh < 2 && ok; ++hh) {
                        const int ko = ko128 + 64 * hh;
                        const int cls = classify_tile64(it.qo, dsf, dsl, ko, P.nc);
                        if (cls == TILE_SKIP) continue;
                        const uint32_t b = sb;
                        sb ^= 1;
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full + 8 * b, (s_phase >> b) & 1u, abort_flag));
                        if (!ok) break;
                        s_phase ^= 1u << b;
                        tc_fence_after();
                        const uint32_t tS = tmem + lane_off + 64 * b;
                        float sf[64];
                        tmem_ld32f(tS, sf);
                        tmem_ld32f(tS + 32, sf + 32);
                        tmem_wait_ld();
                        reg_fence32f(sf);
                        reg_fence32f(sf + 32);
                        if (cls == TILE_PARTIAL) {
                            const int lo = ds_row - ko, hi = q_orig + P.nc - ko;
#pragma unroll
                            for (int c = 0; c < 64; ++c)
                                if (c < lo || c > hi) sf[c] = -INFINITY;
                        }
                        float mx4[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(sf[i], sf[i + 4]);
#pragma unroll
                        for (int c = 8; c < 64; c += 8)
#pragma unroll
                            for (int i = 0; i < 4; ++i) mx4[i] = fmax3(mx4[i], sf[c + i], sf[c + 4 + i]);
                        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                        const float m_tile = mx * P.scale_log2;
                        // lazy rescale: keep the reference max unless it is exceeded by
                        // more than 8 (a factor 256 in the exponentials), or is still -inf
                        const bool need = m_tile > m_used + 8.0f;
                        float alpha = 1.f;
                        if (need) {
                            alpha = ex2_approx(m_used - m_tile);   // 0 when m_used = -inf
                            m_used = m_tile;
                        }
                        const float msub = (m_used == -INFINITY) ? 0.f : m_used;
                        uint32_t pk[32];
                        const float rs = exp_pack64(sf, P.scale_log2, msub, pk);
                        tmem_st32(tS, pk);                  // P over this buffer's S
                        l_sum = l_sum * alpha + rs;
                        if (!first) {
                            // the previous tile's P V has completed: O may be rescaled
                            ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, o_phase, abort_flag));
                            if (!ok) break;
                            o_phase ^= 1;
                            tc_fence_after();
                            if (__any_sync(0xffffffffu, need)) {
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
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_full + 8 * b);
                        first = false;
                        had = true;
                    }
                }
                if (!ok) break;
                if (!P.fused || s == P.s1 - 1) {
                    // ---- epilogue of the segment
                    if (had) {
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, o_phase, abort_flag));
                        if (!ok) break;
                        o_phase ^= 1;
                        tc_fence_after();
                        const bool empty = !(l_sum > 0.f);
                        const float inv_l = empty ? 0.f : 1.f / l_sum;
                        const float lse_v = empty ? -INFINITY
                                                  : (m_used + lg2_approx(l_sum)) * 0.69314718055994531f;
#pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            float of[32];
                            tmem_ld32f(tO + c0, of);
                            tmem_wait_ld();
                            reg_fence32f(of);
                            if (P.fused) {
                                uint4* dst = reinterpret_cast<uint4*>(P.o + rowi * D + c0);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    uint4 u;
                                    u.x = pack_bf16(of[8 * i + 0] * inv_l, of[8 * i + 1] * inv_l);
                                    u.y = pack_bf16(of[8 * i + 2] * inv_l, of[8 * i + 3] * inv_l);
                                    u.z = pack_bf16(of[8 * i + 4] * inv_l, of[8 * i + 5] * inv_l);
                                    u.w = pack_bf16(of[8 * i + 6] * inv_l, of[8 * i + 7] * inv_l);
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
                                    dst[i * step] = make_float4(of[4 * i + 0] * inv_l, of[4 * i + 1] * inv_l,
                                                                of[4 * i + 2] * inv_l, of[4 * i + 3] * inv_l);
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

    // -------------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_relinquish();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace cpattn
