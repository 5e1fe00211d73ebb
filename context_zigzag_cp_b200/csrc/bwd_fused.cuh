// One-pass backward: dK, dV and dQ from a single recomputation of S and dP.
//
// A CTA takes a zigzag pair of 128-key tiles of one KV head (as the dK/dV
// pass: original tiles p and nkt - 1 - p, which together attend to the same
// number of query tiles whatever p is) and, for each key tile, visits every
// query tile of the group's query heads that attends to it.  Per query tile:
//
//     S^T  = K Q^T              -> tensor memory  [0, 128)
//     dP^T = V dO^T             -> tensor memory  [128, 256)
//     P^T  = exp(scale S^T - LSE),  dS^T = P^T (dP^T - delta)     (registers)
//     P^T, dS^T as bf16 over the S^T columns; dS (query-major) to shared memory
//     dV  += P^T dO             (A from tensor memory)             [256, 256+D)
//     dK  += dS^T Q             (A from tensor memory)             [384, 384+D)
//     dQp  = dS K               (A from shared memory) -> the dP^T columns
//     dQ[q rows] += dQp         (fp32 reductions into a global accumulator)
//
// So each (query tile, key tile) pair costs five tile products (the two-pass
// backward pays seven: S and dP again in the dQ pass) plus one fp32 reduction
// of a 128 x D tile.  dQ's accumulator is zeroed by bwd_prep_kernel and scaled
// and rounded to bf16 by dq_convert_kernel; the reductions make dQ's fp32 sum
// order (not its value, beyond rounding) depend on scheduling.
//
// Tensor memory is the constraint that sets the order: the S^T columns hold
// P^T / dS^T until dV and dK have read them, and the dP^T columns hold the dQ
// partial until the elementwise warps have read it out, so per query tile the
// tensor pipe runs S^T, dP^T (once the previous dQ partial is read out), then
// dV, dK, dQp (once P^T, dS^T and dS are written).
//
// The dS tile in shared memory, [128 keys][128 queries] bf16 in two 64-query
// halves with the 128-byte swizzle TMA uses, is the MN-major A operand of
// dQp = dS K; K is its MN-major B operand (as V is for P V in the forward).
#pragma once
#include "bwd.cuh"

namespace cpattn {

template <int D>
struct FusedCfg {
    static constexpr int TILE = 128 * D * 2;
    static constexpr int NQ = 2, NDO = 2;
    static constexpr int K_OFF = 0, V_OFF = TILE;
    static constexpr int Q_OFF = 2 * TILE;
    static constexpr int DO_OFF = Q_OFF + NQ * TILE;
    static constexpr int DS_OFF = DO_OFF + NDO * TILE;            // 128 x 128 bf16, two halves
    static constexpr int DS_BYTES = 128 * 128 * 2;
    static constexpr int LQ_OFF = DS_OFF + DS_BYTES;              // nlse2 rows [NQ]
    static constexpr int LD_OFF = LQ_OFF + NQ * 512;              // delta rows [NDO]
    static constexpr int BAR_OFF = LD_OFF + NDO * 512;
    // kv_full, kv_empty, q_full[NQ], q_empty[NQ], do_full[NDO], do_empty[NDO], st_ready, dp_ready,
    // p_full, dq_ready, dq_free, acc_full, acc_empty, drain
    static constexpr int NBAR = 9 + 2 * NQ + 2 * NDO;
    // the dynamic shared window starts 1024-byte aligned (checked at run time), no slack
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64;
    static constexpr int THREADS = BWD_THREADS;
};

// dQ accumulator -> bf16 dQ: dq[i] = bf16(scale * acc[i]), 8 values per thread step.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ acc,
                                                         uint4* __restrict__ dq, int64_t n8, float scale)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 a = __ldg(acc + 2 * i), b = __ldg(acc + 2 * i + 1);
        dq[i] = make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                           pack_bf16(b.x * scale, b.y * scale), pack_bf16(b.z * scale, b.w * scale));
    }
}

template <int D, bool PD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
cp_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams P)
{
    using Cfg = FusedCfg<D>;
    constexpr bool kDqT = (D == 128);   // the dQ partial transposed (head-dim on the lanes)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023u) {   // swizzled tiles need a 1024-byte aligned window
        if (threadIdx.x == 0) record_status(3 /* CP_ERR_CUDA */);
        return;
    }
    uint8_t* smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sK = sbase + Cfg::K_OFF, sV = sbase + Cfg::V_OFF;
    const uint32_t sQ = sbase + Cfg::Q_OFF, sdO = sbase + Cfg::DO_OFF, sDS = sbase + Cfg::DS_OFF;
    const uint32_t sLQ = sbase + Cfg::LQ_OFF, sLD = sbase + Cfg::LD_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_kv_full = bars, bar_kv_empty = bars + 8;
    const uint32_t bar_q_full = bars + 16, bar_q_empty = bar_q_full + 8 * Cfg::NQ;
    const uint32_t bar_do_full = bar_q_empty + 8 * Cfg::NQ, bar_do_empty = bar_do_full + 8 * Cfg::NDO;
    const uint32_t bar_st_ready = bar_do_empty + 8 * Cfg::NDO, bar_dp_ready = bar_st_ready + 8;
    const uint32_t bar_p_full = bar_dp_ready + 8, bar_dq_ready = bar_p_full + 8;
    const uint32_t bar_dq_free = bar_dq_ready + 8, bar_acc_full = bar_dq_free + 8;
    const uint32_t bar_acc_empty = bar_acc_full + 8, bar_drain = bar_acc_empty + 8;
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
        mbar_init(bar_p_full, 4 * BWD_NWG);
        mbar_init(bar_dq_ready, 1);
        mbar_init(bar_dq_free, 4 * BWD_NWG);
        mbar_init(bar_acc_full, 1);
        mbar_init(bar_acc_empty, 4 * BWD_NWG);
        mbar_init(bar_drain, 1);
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
                if (!(P.stall == 12 /* CP_K_BWD_FUSED */ && blockIdx.x == 0 && iter == 0)) {
                    mbar_arrive_expect_tx(bar_kv_full, 2 * Cfg::TILE);
                    const int kvrow = it.bkv * P.kv_rows + it.krow;
                    for (int h = 0; h < D / 64; ++h) {
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
        // of tensor-core instructions.
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);   // K-major A and B
            constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);      // A tmem, B MN-major
            // dQ partial: at D = 128 transposed, dQp^T = K^T dS^T (head-dim on the TMEM lanes,
            // so the reduction of a query row is one coalesced line per warp); at D = 64 as
            // dQp = dS K (an M = 64 accumulator would use half the lanes)
            constexpr uint32_t IDESC_Q = kDqT ? idesc_bf16(128, 128, true, true)
                                              : idesc_bf16(128, D, true, true);   // A, B MN-major
            constexpr uint32_t TILE16 = Cfg::TILE >> 4;
            const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
            // descriptor bases; k-steps and stages are constant offsets in 16-byte units
            const uint64_t dK = sdesc_sw128(sK, 16, 1024), dVk = sdesc_sw128(sV, 16, 1024);
            const uint64_t dKmn = sdesc_sw128(sK, 16384, 1024);
            const uint64_t dQk = sdesc_sw128(sQ, 16, 1024), dQmn = sdesc_sw128(sQ, 16384, 1024);
            const uint64_t dOk = sdesc_sw128(sdO, 16, 1024), dOmn = sdesc_sw128(sdO, 16384, 1024);
            const uint64_t dDSmn = sdesc_sw128(sDS, 16384, 1024);
            uint32_t nst = 0, iter = 0, p_phase = 0, df_phase = 0, ae_phase = 0;
            // acc_busy: the last item's accumulators not yet read out; dq_pending: a dQ
            // partial sits in the dP^T columns and has not been read out yet
            bool ok = true, acc_busy = false, dq_pending = false;
            for (int w = blockIdx.x; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
                const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
                ok = mbar_wait_warp(bar_kv_full, iter & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool first = true;
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
                        tc_fence_after();
                        const uint64_t bq = dQk + qs * TILE16, bdo = dOk + ds * TILE16;
                        // S^T: the S^T columns are free once the previous tile's dV / dK were
                        // issued (the tensor pipe runs in order)
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ss(tS, dK + off, bq + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_st_ready);
                        }
                        __syncwarp();
                        ok = mbar_wait_warp(bar_do_full + 8 * ds, dpar, abort_flag);
                        if (!ok) break;
                        if (dq_pending) {   // the previous dQ partial has been read out of the dP^T columns
                            ok = mbar_wait_warp(bar_dq_free, df_phase, abort_flag);
                            if (!ok) break;
                            df_phase ^= 1;
                            dq_pending = false;
                        }
                        tc_fence_after();
                        if (elect_one()) {
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint32_t off = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                mma_ss(tdP, dVk + off, bdo + off, IDESC_S, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_dp_ready);
                        }
                        __syncwarp();
                        if (first && acc_busy) {   // every group has stored the previous item's dK / dV
                            ok = mbar_wait_warp(bar_acc_empty, ae_phase, abort_flag);
                            if (!ok) break;
                            ae_phase ^= 1;
                            acc_busy = false;
                        }
                        // P^T / dS^T in the S^T columns and dS in shared memory
                        ok = mbar_wait_warp(bar_p_full, p_phase, abort_flag);
                        if (!ok) break;
                        p_phase ^= 1;
                        tc_fence_after();
                        const uint64_t bq_mn = dQmn + qs * TILE16, bdo_mn = dOmn + ds * TILE16;
                        if (elect_one()) {
                            // dV += P^T dO and dK += dS^T Q: k-step (j, w4) covers queries
                            // 64j + 16w4 .. +15, whose P^T / dS^T sit at S^T columns
                            // 64j + 16w4 (+8 for dS^T)
#pragma unroll
                            for (int j = 0; j < 2; ++j)
#pragma unroll
                                for (int w4 = 0; w4 < 4; ++w4) {
                                    const uint32_t acc = (!first || j > 0 || w4 > 0) ? 1u : 0u;
                                    const uint32_t brow = ((4 * j + w4) * 2048) >> 4;
                                    mma_ts(tdV, tS + 64 * j + 16 * w4, bdo_mn + brow, IDESC_G, acc);
                                    mma_ts(tdK, tS + 64 * j + 16 * w4 + 8, bq_mn + brow, IDESC_G, acc);
                                }
                            // the dQ partial into the dP^T columns (dP^T was read before dS was
                            // formed): K^T (MN-major A) dS^T (MN-major B), or dS (A) K (B)
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const uint32_t ks = (k * 2048) >> 4;
                                if (kDqT) mma_ss(tdP, dKmn + ks, dDSmn + ks, IDESC_Q, k > 0 ? 1u : 0u);
                                else mma_ss(tdP, dDSmn + ks, dKmn + ks, IDESC_Q, k > 0 ? 1u : 0u);
                            }
                            mma_commit(bar_dq_ready);
                            mma_commit(bar_q_empty + 8 * qs);
                            mma_commit(bar_do_empty + 8 * ds);
                        }
                        __syncwarp();
                        dq_pending = true;
                        first = false;
                    }
                }
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
        const uint32_t tdQ = tmem + lane_off + 128 + 32 * wg;   // dQ partial: 32 of its D columns
        // this thread's dS row in shared memory: key row `row`, queries 64j + 16wg .. +15,
        // i.e. 16-byte chunks 2wg and 2wg+1 of row `row` of half j (128-byte swizzle)
        uint8_t* ds_row = smem + Cfg::DS_OFF + row * 128;
        const int ch0 = ((2 * wg) ^ (row & 7)) * 16, ch1 = ((2 * wg + 1) ^ (row & 7)) * 16;
        uint32_t nst = 0, st_phase = 0, dp_phase = 0, dq_phase = 0, a_phase = 0;
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
                    const int bh = it.b * P.Hq + it.hk * g + hq;
                    const float* s_nlse2 = reinterpret_cast<const float*>(smem + Cfg::LQ_OFF + qs * 512) + 16 * wg;
                    const float* s_delta = reinterpret_cast<const float*>(smem + Cfg::LD_OFF + ds * 512) + 16 * wg;
                    const int* s_ds = P.doc_start + qpos + 16 * wg;   // documents only (global, cached)
                    // ---- S^T: copy out and form P^T while dP^T is being computed
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_st_ready, st_phase, abort_flag));
                    if (!ok) break;
                    st_phase ^= 1;
                    tc_fence_after();
                    float sv[32], dp[32];
                    tmem_ld16f(tS, sv);
                    tmem_ld16f(tS + 64, sv + 16);
                    tmem_wait_ld();
                    reg_fence32f(sv);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
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
                    // ---- dP^T: copy out, form dS^T, write P^T / dS^T over this warp's own
                    // S^T columns (already read) and dS into shared memory
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_ready, dp_phase, abort_flag));
                    if (!ok) break;
                    dp_phase ^= 1;
                    tc_fence_after();
                    tmem_ld16f(tdP, dp);
                    tmem_ld16f(tdP + 64, dp + 16);
                    tmem_wait_ld();
                    reg_fence32f(dp);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        uint32_t pk[8], dk[8];
                        dkdv_ds16(sv + 16 * j, dp + 16 * j, s_delta + 64 * j, pk, dk);
                        tmem_st8(tS + 64 * j, pk);
                        tmem_st8(tS + 64 * j + 8, dk);
                        uint8_t* half = ds_row + j * (Cfg::DS_BYTES / 2);
                        *reinterpret_cast<uint4*>(half + ch0) = make_uint4(dk[0], dk[1], dk[2], dk[3]);
                        *reinterpret_cast<uint4*>(half + ch1) = make_uint4(dk[4], dk[5], dk[6], dk[7]);
                    }
                    tmem_wait_st();
                    // generic-proxy writes of dS -> visible to the tensor core (async proxy)
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_p_full);
                    // ---- dQ partial (query rows on the TMEM lanes): read out, release the
                    // columns, then reduce into the fp32 accumulator
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dq_ready, dq_phase, abort_flag));
                    if (!ok) break;
                    dq_phase ^= 1;
                    tc_fence_after();
                    float qa[32];
                    if (kDqT || 32 * wg < D) {
                        tmem_ld32f(tdQ, qa);
                        tmem_wait_ld();
                        reg_fence32f(qa);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_dq_free);
                    if (kDqT) {
                        // lane `row` holds head-dim column d = row of query rows 32wg .. 32wg+31:
                        // a warp's 32 lanes add one contiguous 128-byte line per query row
                        const size_t qrow0 = static_cast<size_t>(bh) * P.q_rows + (qpos - P.q_base) + 32 * wg;
                        float* dst = P.dq_acc + qrow0 * D + row;
#pragma unroll
                        for (int i = 0; i < 32; ++i) atomicAdd(dst + static_cast<size_t>(i) * D, qa[i]);
                    } else if (32 * wg < D) {
                        const size_t qrow = static_cast<size_t>(bh) * P.q_rows + (qpos - P.q_base) + row;
                        float4* dst = reinterpret_cast<float4*>(P.dq_acc + qrow * D + 32 * wg);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            atomicAdd(dst + i, make_float4(qa[4 * i], qa[4 * i + 1], qa[4 * i + 2], qa[4 * i + 3]));
                    }
                    had = true;
                }
            }
            if (!ok) break;
            // ---- epilogue: this group's 32 columns of dK (scaled) and dV
            const size_t orow = static_cast<size_t>(it.bkv) * P.S + it.kpos + row;
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
                            dv[i] = make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
                            dk[i] = make_float4(b[4 * i] * P.scale, b[4 * i + 1] * P.scale,
                                                b[4 * i + 2] * P.scale, b[4 * i + 3] * P.scale);
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
            } else if (32 * wg < D) {
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

}  // namespace cpattn
