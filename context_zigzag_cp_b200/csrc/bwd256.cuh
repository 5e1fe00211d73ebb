// Backward at head_dim 256: dQ, dK, dV from the final LSE, the same
// computation as the head_dim-128 passes, in three passes.
//
// At D = 256 the dK and dV accumulators of a 128-key tile (256 fp32 columns
// each) would fill all 512 tensor-memory columns with no room left for S^T and
// dP^T, so dV and dK get a pass each (the two instantiations of
// cp_bwd256_kv_kernel) besides the dQ pass (cp_bwd256_dq_kernel); S is
// recomputed in each, dP in the dK and dQ passes.  Work units are 64 rows wide
// on the side that streams (64-query units against a 128-key tile; 64-key tiles
// against a 128-row query tile), so the operand tiles fit shared memory next to
// the resident ones, and the schedule is the head_dim-128 one: the elementwise
// warps copy S out and release it, the tensor core computes the next tile's S
// while they form P, and the products of a finished tile read P / dS (bf16)
// from tensor memory.
#pragma once
#include "bwd.cuh"
#include "fwd256.cuh"

namespace cpattn {

// A 64-row query unit [qo, qo+63] (first visible keys dsf..dsl over its rows)
// against the 128-key tile [ko, ko+127].
__device__ __forceinline__ int classify_q64(int qo, int dsf, int dsl, int ko, int nc)
{
    if (ko > qo + 63 + nc || ko + 127 < dsf) return TILE_SKIP;
    if (ko + 127 <= qo + nc && ko >= dsl) return TILE_FULL;
    return TILE_PARTIAL;
}

// 16 fp32 values packed to 8 bf16 pairs.
__device__ __forceinline__ void pack16(const float* v, uint32_t* pk)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
}

// ============================================================================
// dV pass (MODE 0) and dK pass (MODE 1)
// ============================================================================
// Per 128-key tile (the dK/dV pass's zigzag pairs of key tiles), every
// attending 64-row query unit of every query head of the GQA group:
//   S^T = K Q^T            (SS: K resident, Q unit streamed)      -> TMEM [0, 64)
//   MODE 0: P^T (bf16) into TMEM [64, 96) / [96, 128) (alternating units);
//           dV += P^T dO   (A from TMEM, dO unit MN-major)        -> TMEM [256, 512)
//   MODE 1: dP^T = V dO^T  (SS: V resident)                       -> TMEM [64, 128)
//           dS^T (bf16) over the dP^T columns each warp has read;
//           dK += dS^T Q   (A from TMEM, Q unit MN-major)         -> TMEM [256, 512)
// Shared memory: the K tile (and the V tile), rings of Q and dO units (32 KB
// each).  The units' -LSE*log2(e) (and delta) values are read by the
// elementwise warps from global memory into registers (16 per warp, the same
// for its 32 rows, so L1 serves them), ahead of the wait for S^T: a ring slot
// is released when its tile's last product is issued, which can be before the
// elementwise step of that unit has ended.
template <int MODE>
struct Kv256Cfg {
    static constexpr int D = 256;
    static constexpr int KTILE = 128 * D * 2;          // resident K / V tile: four 16 KB boxes
    static constexpr int QT = 64;                       // query rows per unit
    static constexpr int QTILE = QT * D * 2;            // 32 KB: four 8 KB boxes
    static constexpr int QBOX = QT * 128;
    static constexpr int NQ = MODE == 0 ? 3 : 2, NDO = MODE == 0 ? 2 : 1;
    static constexpr int K_OFF = 0, V_OFF = KTILE;      // V only in MODE 1
    static constexpr int Q_OFF = (MODE == 0 ? 1 : 2) * KTILE;
    static constexpr int DO_OFF = Q_OFF + NQ * QTILE;
    static constexpr int BAR_OFF = DO_OFF + NDO * QTILE;
    // kv_full, kv_empty, q_full[NQ], q_empty[NQ], do_full[NDO], do_empty[NDO], st_ready,
    // dp_ready, s_free, p_full[2], acc_full, drain, acc_empty
    static constexpr int NBAR = 10 + 2 * NQ + 2 * NDO;
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64 + 1024;   // + alignment slack
    static constexpr int THREADS = BWD_THREADS;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

template <bool PD, int MODE>
__global__ void __launch_bounds__(BWD_THREADS, 1)
cp_bwd256_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams P)
{
    using Cfg = Kv256Cfg<MODE>;
    constexpr int D = Cfg::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sK = sbase + Cfg::K_OFF, sV = sbase + Cfg::V_OFF;
    const uint32_t sQ = sbase + Cfg::Q_OFF, sdO = sbase + Cfg::DO_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_kv_full = bars, bar_kv_empty = bars + 8;
    const uint32_t bar_q_full = bars + 16, bar_q_empty = bar_q_full + 8 * Cfg::NQ;
    const uint32_t bar_do_full = bar_q_empty + 8 * Cfg::NQ, bar_do_empty = bar_do_full + 8 * Cfg::NDO;
    const uint32_t bar_st_ready = bar_do_empty + 8 * Cfg::NDO, bar_dp_ready = bar_st_ready + 8;
    // p_full[u & 1] for unit u: in the dV pass nothing orders the elementwise step of
    // unit u+1 after the MMA warp's wait for unit u (S^T(u+1) is issued first), so one
    // barrier could complete twice before that wait and its parity would alias
    const uint32_t bar_s_free = bar_dp_ready + 8, bar_p_full = bar_s_free + 8;   // [2]
    const uint32_t bar_acc_full = bar_p_full + 16, bar_drain = bar_acc_full + 8;
    const uint32_t bar_acc_empty = bar_drain + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::BAR_OFF + Cfg::NBAR * 8 + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.Hq / P.Hkv;
    const int ntq = P.S / 128;
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
        mbar_init(bar_p_full, 4 * BWD_NWG);
        mbar_init(bar_p_full + 8, 4 * BWD_NWG);
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
      regs_dec<64>();
      if (warp == PROD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmdO);
            if (MODE == 1) prefetch_tmap(&tmV);
            uint32_t nst = 0, iter = 0;
            bool ok = true, kv_issued = false;
            for (int w = blockIdx.x; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
                const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
                ok = mbar_wait(bar_kv_empty, (iter & 1) ^ 1, abort_flag);
                if (!ok) break;
                kv_issued = true;
                // test hook (cp_selftest_stall): the first K/V tile of CTA 0 is never loaded
                if (!(P.stall == 7 /* CP_K_BWD_DKDV */ && blockIdx.x == 0 && iter == 0)) {
                    mbar_arrive_expect_tx(bar_kv_full, (MODE == 1 ? 2 : 1) * Cfg::KTILE);
                    const int kvrow = it.bkv * P.kv_rows + it.krow;
                    for (int h = 0; h < D / 64; ++h) {
                        tma_load_2d(sK + h * 16384, &tmK, h * 64, kvrow, bar_kv_full);
                        if (MODE == 1) tma_load_2d(sV + h * 16384, &tmV, h * 64, kvrow, bar_kv_full);
                    }
                }
                const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
                for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                    const int tq = abs(u);
                    const int qpos128 = shard_of_tile<PD>(P, tq * 128);
                    for (int qh = 0; qh < 2 && ok; ++qh) {
                        const int qo = tq * 128 + 64 * qh, qpos = qpos128 + 64 * qh;
                        const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                        const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 63) : 0, qo + 63 - P.wm1);
                        if (classify_q64(qo, dsf, dsl, it.ko, P.nc) == TILE_SKIP || !q_tile_on_rank(P, qpos))
                            continue;
                        for (int hq = 0; hq < g && ok; ++hq) {
                            const int bh = it.b * P.Hq + it.hk * g + hq;
                            const size_t row = static_cast<size_t>(bh) * P.q_rows + (qpos - P.q_base);
                            const uint32_t qs = nst % Cfg::NQ, qp = (nst / Cfg::NQ) & 1;
                            const uint32_t ds = nst % Cfg::NDO, dpar = (nst / Cfg::NDO) & 1;
                            ++nst;
                            ok = mbar_wait(bar_q_empty + 8 * qs, qp ^ 1, abort_flag);
                            if (!ok) break;
                            mbar_arrive_expect_tx(bar_q_full + 8 * qs, Cfg::QTILE);
                            for (int h = 0; h < D / 64; ++h)
                                tma_load_2d(sQ + qs * Cfg::QTILE + h * Cfg::QBOX, &tmQ, h * 64,
                                            static_cast<int>(row), bar_q_full + 8 * qs);
                            ok = mbar_wait(bar_do_empty + 8 * ds, dpar ^ 1, abort_flag);
                            if (!ok) break;
                            mbar_arrive_expect_tx(bar_do_full + 8 * ds, Cfg::QTILE);
                            for (int h = 0; h < D / 64; ++h)
                                tma_load_2d(sdO + ds * Cfg::QTILE + h * Cfg::QBOX, &tmdO, h * 64,
                                            static_cast<int>(row), bar_do_full + 8 * ds);
                        }
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
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, Cfg::QT, false, false);   // K-major A and B
            constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);         // A tmem, B MN-major
            constexpr uint32_t QT16 = Cfg::QTILE >> 4;
            const uint32_t tS = tmem, tX = tmem + 64, tAcc = tmem + 256;
            const uint64_t dKk = sdesc_sw128(sK, 16, 1024), dVk = sdesc_sw128(sV, 16, 1024);
            const uint64_t dQk = sdesc_sw128(sQ, 16, 1024), dQmn = sdesc_sw128(sQ, Cfg::QBOX, 1024);
            const uint64_t dOk = sdesc_sw128(sdO, 16, 1024), dOmn = sdesc_sw128(sdO, Cfg::QBOX, 1024);
            uint32_t nst = 0, iter = 0, sf_phase = 0, ae_phase = 0;
            uint32_t p_phase = 0;             // bit b: parity of the next wait on p_full[b]
            bool ok = true, acc_busy = false, s_pending = false;
            // the products of one finished unit: MODE 0 dV += P^T dO (P^T at columns 64 + 32pb,
            // query rows 16w .. +15 at + 8w); MODE 1 dK += dS^T Q (dS^T over the dP^T columns,
            // query rows 16w .. +15 at 64 + 16w)
            auto issue_products = [&](uint32_t qs, uint32_t ds, uint32_t dpar, uint32_t pb, bool& first) -> bool {
                if (first && acc_busy) {   // every group has stored the previous item's accumulator
                    if (!mbar_wait_warp(bar_acc_empty, ae_phase, abort_flag)) return false;
                    ae_phase ^= 1;
                    acc_busy = false;
                }
                if (!mbar_wait_warp(bar_p_full + 8 * pb, (p_phase >> pb) & 1u, abort_flag)) return false;
                p_phase ^= 1u << pb;
                // MODE 0: the unit's dO (MODE 1 waited for it before its dP^T)
                if (MODE == 0 && !mbar_wait_warp(bar_do_full + 8 * ds, dpar, abort_flag)) return false;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {
                        const uint32_t acc = (!first || w4 > 0) ? 1u : 0u;
                        const uint32_t brow = (w4 * 2048) >> 4;
                        if (MODE == 0)
                            mma_ts(tAcc, tX + 32 * pb + 8 * w4, dOmn + ds * QT16 + brow, IDESC_G, acc);
                        else
                            mma_ts(tAcc, tX + 16 * w4, dQmn + qs * QT16 + brow, IDESC_G, acc);
                    }
                    if (MODE == 0) mma_commit(bar_do_empty + 8 * ds);
                    else mma_commit(bar_q_empty + 8 * qs);
                }
                __syncwarp();
                first = false;
                return true;
            };
            for (int w = blockIdx.x; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
                const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
                ok = mbar_wait_warp(bar_kv_full, iter & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool first = true, prev_live = false;
                uint32_t prev_qs = 0, prev_ds = 0, prev_dpar = 0, prev_pb = 0;
                const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
                for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                    const int tq = abs(u);
                    const int qpos128 = shard_of_tile<PD>(P, tq * 128);
                    for (int qh = 0; qh < 2 && ok; ++qh) {
                        const int qo = tq * 128 + 64 * qh, qpos = qpos128 + 64 * qh;
                        const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                        const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 63) : 0, qo + 63 - P.wm1);
                        if (classify_q64(qo, dsf, dsl, it.ko, P.nc) == TILE_SKIP || !q_tile_on_rank(P, qpos))
                            continue;
                        for (int hq = 0; hq < g && ok; ++hq) {
                            const uint32_t qs = nst % Cfg::NQ, qp = (nst / Cfg::NQ) & 1;
                            const uint32_t ds = nst % Cfg::NDO, dpar = (nst / Cfg::NDO) & 1;
                            const uint32_t pb = nst & 1;
                            ++nst;
                            ok = mbar_wait_warp(bar_q_full + 8 * qs, qp, abort_flag);
                            if (!ok) break;
                            if (s_pending) {   // the previous unit's S^T (and dP^T) are copied out
                                ok = mbar_wait_warp(bar_s_free, sf_phase, abort_flag);
                                if (!ok) break;
                                sf_phase ^= 1;
                            }
                            tc_fence_after();
                            // S^T of this unit while the elementwise warps still work on the previous one
                            if (elect_one()) {
                                const uint64_t bq = dQk + qs * QT16;
#pragma unroll
                                for (int k = 0; k < D / 16; ++k) {
                                    const uint32_t offa = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                    const uint32_t offb = ((k / 4) * Cfg::QBOX + (k % 4) * 32) >> 4;
                                    mma_ss(tS, dKk + offa, bq + offb, IDESC_S, k > 0 ? 1u : 0u);
                                }
                                mma_commit(bar_st_ready);
                                if (MODE == 0) mma_commit(bar_q_empty + 8 * qs);   // Q only feeds S^T
                            }
                            __syncwarp();
                            s_pending = true;
                            // the previous unit's products read P^T / dS^T from tensor memory ...
                            if (prev_live && !(ok = issue_products(prev_qs, prev_ds, prev_dpar, prev_pb, first))) break;
                            if (MODE == 1) {
                                // ... before this unit's dP^T overwrites them (the tensor pipe runs in order)
                                ok = mbar_wait_warp(bar_do_full + 8 * ds, dpar, abort_flag);
                                if (!ok) break;
                                tc_fence_after();
                                if (elect_one()) {
                                    const uint64_t bdo = dOk + ds * QT16;
#pragma unroll
                                    for (int k = 0; k < D / 16; ++k) {
                                        const uint32_t offa = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                        const uint32_t offb = ((k / 4) * Cfg::QBOX + (k % 4) * 32) >> 4;
                                        mma_ss(tX, dVk + offa, bdo + offb, IDESC_S, k > 0 ? 1u : 0u);
                                    }
                                    mma_commit(bar_dp_ready);
                                    mma_commit(bar_do_empty + 8 * ds);
                                }
                                __syncwarp();
                            }
                            prev_live = true;
                            prev_qs = qs;
                            prev_ds = ds;
                            prev_dpar = dpar;
                            prev_pb = pb;
                        }
                    }
                }
                if (ok && prev_live) ok = issue_products(prev_qs, prev_ds, prev_dpar, prev_pb, first);
                if (!ok) break;
                if (elect_one()) {
                    mma_commit(bar_kv_empty);
                    if (!first) mma_commit(bar_acc_full);   // the elementwise groups wait only if they had a unit
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
        const int wg = warp >> 2;                        // query columns [16wg, 16wg+16) of a unit
        const int row = (warp & 3) * 32 + lane;          // key row of the tile (TMEM lane)
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 16 * wg;
        const uint32_t tdP = tmem + lane_off + 64 + 16 * wg;            // MODE 1
        const uint32_t tPk = tmem + lane_off + 64 + 8 * wg;             // MODE 0, + 32 pb
        const uint32_t tAcc = tmem + lane_off + 256 + 64 * wg;
        uint32_t nst = 0, st_phase = 0, dp_phase = 0, a_phase = 0;
        bool ok = true;
        for (int w = blockIdx.x, iter = 0; w < P.n_items && ok; w = blockIdx.x + ((++iter) >> 1) * gridDim.x) {
            const DkdvItem it = decode_dkdv<PD>(P, w, iter & 1);
            const int k_orig = it.ko + row;
            bool had = false;
            const DkdvWalk wk = dkdv_walk(max(0, it.ko - P.nc) / 128, dkdv_last_tile(P, it.ko, ntq), iter);
            for (int u = wk.u0; u < wk.u1 && ok; ++u) {
                const int tq = abs(u);
                const int qpos128 = shard_of_tile<PD>(P, tq * 128);
                for (int qh = 0; qh < 2 && ok; ++qh) {
                    const int qo = tq * 128 + 64 * qh, qpos = qpos128 + 64 * qh;
                    const int dsf = max(P.docs ? __ldg(P.doc_start + qpos) : 0, qo - P.wm1);
                    const int dsl = max(P.docs ? __ldg(P.doc_start + qpos + 63) : 0, qo + 63 - P.wm1);
                    const int cls = classify_q64(qo, dsf, dsl, it.ko, P.nc);
                    if (cls == TILE_SKIP || !q_tile_on_rank(P, qpos)) continue;
                    for (int hq = 0; hq < g && ok; ++hq) {
                        const uint32_t pb = nst & 1;
                        ++nst;
                        // this warp's 16 query columns: -LSE*log2(e) and delta, ahead of S^T
                        const int bh = it.b * P.Hq + it.hk * g + hq;
                        const size_t urow = static_cast<size_t>(bh) * P.q_rows + (qpos - P.q_base) + 16 * wg;
                        float s_nlse2[16], s_delta[16];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 a = __ldg(reinterpret_cast<const float4*>(P.nlse2 + urow) + i);
                            s_nlse2[4 * i] = a.x; s_nlse2[4 * i + 1] = a.y; s_nlse2[4 * i + 2] = a.z; s_nlse2[4 * i + 3] = a.w;
                            if (MODE == 1) {
                                const float4 b = __ldg(reinterpret_cast<const float4*>(P.delta + urow) + i);
                                s_delta[4 * i] = b.x; s_delta[4 * i + 1] = b.y; s_delta[4 * i + 2] = b.z; s_delta[4 * i + 3] = b.w;
                            } else {
                                s_delta[4 * i] = s_delta[4 * i + 1] = s_delta[4 * i + 2] = s_delta[4 * i + 3] = 0.f;
                            }
                        }
                        const int* s_ds = P.doc_start + qpos + 16 * wg;   // documents only (global, cached)
                        // ---- S^T: copy out, release, and form P^T
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_st_ready, st_phase, abort_flag));
                        if (!ok) break;
                        st_phase ^= 1;
                        tc_fence_after();
                        float sv[16], dp[16];
                        tmem_ld16f(tS, sv);
                        tmem_wait_ld();
                        reg_fence16f(sv);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_s_free);   // the MMA warp may compute the next S^T
                        // column c (query qo + 16wg + c) is admitted when k - nc <= q and
                        // q <= k + wm1: thr - nc <= c <= thr + wm1
                        const int thr = k_orig - (qo + 16 * wg) - P.nc;
                        const int wsp = P.wm1 + P.nc;
                        if (cls == TILE_FULL)
                            dkdv_p16<0>(sv, s_nlse2, s_ds, P.scale_log2, thr, wsp, k_orig);
                        else if (!P.docs)
                            dkdv_p16<1>(sv, s_nlse2, s_ds, P.scale_log2, thr, wsp, k_orig);
                        else
                            dkdv_p16<2>(sv, s_nlse2, s_ds, P.scale_log2, thr, wsp, k_orig);
                        uint32_t pk[8], dk[8];
                        if (MODE == 0) {
                            pack16(sv, pk);
                            tmem_st8(tPk + 32 * pb, pk);
                        } else {
                            // ---- dP^T: copy out; dS^T (bf16) goes over this warp's own columns
                            ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_ready, dp_phase, abort_flag));
                            if (!ok) break;
                            dp_phase ^= 1;
                            tc_fence_after();
                            tmem_ld16f(tdP, dp);
                            tmem_wait_ld();
                            reg_fence16f(dp);
                            dkdv_ds16(sv, dp, s_delta, pk, dk);
                            tmem_st8(tdP, dk);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_full + 8 * pb);
                        had = true;
                    }
                }
            }
            if (!ok) break;
            // ---- epilogue: this group's 64 columns of dV (MODE 0) or dK (MODE 1, scaled)
            const size_t orow = P.step_shard ? static_cast<size_t>(it.bkv) * 2 * P.C + it.krow + row
                                             : static_cast<size_t>(it.bkv) * P.S + it.kpos + row;
            const float mul = MODE == 0 ? 1.f : P.scale;
            float* out32 = MODE == 0 ? P.dv32 : P.dk32;
            __nv_bfloat16* out16 = MODE == 0 ? P.dv : P.dk;
            if (had) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full, a_phase, abort_flag));
                if (!ok) break;
                a_phase ^= 1;
                tc_fence_after();
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float a[32];
                    tmem_ld32f(tAcc + 32 * h, a);
                    tmem_wait_ld();
                    reg_fence32f(a);
                    const size_t col = 64 * wg + 32 * h;
                    if (out32) {   // fp32 partials (one rank's share, summed across ranks later)
                        float4* dst = reinterpret_cast<float4*>(out32 + orow * D + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float4 x = make_float4(a[4 * i] * mul, a[4 * i + 1] * mul, a[4 * i + 2] * mul,
                                                   a[4 * i + 3] * mul);
                            if (P.accumulate) {   // this CTA owns the rows: a plain read-modify-write
                                const float4 u = dst[i];
                                x.x += u.x; x.y += u.y; x.z += u.z; x.w += u.w;
                            }
                            dst[i] = x;
                        }
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(out16 + orow * D + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pack_bf16(a[8 * i] * mul, a[8 * i + 1] * mul),
                                                pack_bf16(a[8 * i + 2] * mul, a[8 * i + 3] * mul),
                                                pack_bf16(a[8 * i + 4] * mul, a[8 * i + 5] * mul),
                                                pack_bf16(a[8 * i + 6] * mul, a[8 * i + 7] * mul));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty);
            } else if (P.accumulate) {
                // nothing to add
            } else if (out32) {
                float4* dst = reinterpret_cast<float4*>(out32 + orow * D + 64 * wg);
                for (int i = 0; i < 16; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(out16 + orow * D + 64 * wg);
                for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
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
// Per 128-row query tile and every visible 64-key tile, in the plan's visit
// order:  S = Q K^T (A: the tile's Q rows in TMEM [128, 256)) -> TMEM [0, 64);
// dP = dO V^T (SS: the tile's dO resident in shared memory) -> TMEM [64, 128);
// dS (bf16) over the dP columns each warp has read; dQ += dS K (A from TMEM,
// K MN-major) -> TMEM [256, 512).  Shared memory: the dO tile (64 KB) and a
// 5-slot ring of 64-row K / V tiles.
struct Dq256Cfg {
    static constexpr int D = 256, KT = 64;
    static constexpr int KTILE = KT * D * 2;            // 32 KB K or V tile: four 8 KB boxes
    static constexpr int KBOX = KT * 128;
    static constexpr int DO_BYTES = 128 * D * 2;        // 64 KB dO tile: four 16 KB boxes
    static constexpr int NSLOT = 5;
    static constexpr int DO_OFF = 0, KV_OFF = DO_BYTES;
    static constexpr int BAR_OFF = KV_OFF + NSLOT * KTILE;
    // qt_full, qt_empty, do_full, kv_full[NSLOT], kv_empty[NSLOT], st_ready, dp_ready, s_free,
    // p_full, acc_full, drain, acc_empty
    static constexpr int NBAR = 10 + 2 * NSLOT;
    static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 64 + 1024;   // + alignment slack
    static constexpr int THREADS = BWD_THREADS;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

template <bool PD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
cp_bwd256_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmdO, const BwdParams P)
{
    using Cfg = Dq256Cfg;
    constexpr int D = Cfg::D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sdO = sbase + Cfg::DO_OFF, sKV = sbase + Cfg::KV_OFF;
    const uint32_t bars = sbase + Cfg::BAR_OFF;
    const uint32_t bar_qt_full = bars, bar_qt_empty = bars + 8, bar_do_full = bars + 16;
    const uint32_t bar_kv_full = bars + 24, bar_kv_empty = bars + 24 + 8 * Cfg::NSLOT;
    const uint32_t bar_st_ready = bars + 24 + 16 * Cfg::NSLOT, bar_dp_ready = bar_st_ready + 8;
    const uint32_t bar_s_free = bar_dp_ready + 8, bar_p_full = bar_s_free + 8;
    const uint32_t bar_acc_full = bar_p_full + 8, bar_drain = bar_acc_full + 8;
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
        mbar_init(bar_do_full, 1);
        for (int i = 0; i < Cfg::NSLOT; ++i) {
            mbar_init(bar_kv_full + 8 * i, 1);
            mbar_init(bar_kv_empty + 8 * i, 1);
        }
        mbar_init(bar_st_ready, 1);
        mbar_init(bar_dp_ready, 1);
        mbar_init(bar_s_free, 4 * BWD_NWG);
        mbar_init(bar_p_full, 4 * BWD_NWG);
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
      regs_dec<64>();
      if (warp == PROD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmdO);
            uint32_t nload = 0, iter = 0;
            bool ok = true, do_issued = false;
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const DqItem it = decode_dq<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                // the tile's dO, once the previous item's dP products have read the old one
                ok = mbar_wait(bar_qt_empty, (iter & 1) ^ 1, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(bar_do_full, Cfg::DO_BYTES);
                do_issued = true;
                const int drow = static_cast<int>(static_cast<size_t>(it.bh) * P.q_rows + (it.qpos - P.q_base));
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(sdO + h * 16384, &tmdO, h * 64, drow, bar_do_full);
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
                                const uint32_t slot = nload % Cfg::NSLOT, par = (nload / Cfg::NSLOT) & 1;
                                ok = mbar_wait(bar_kv_empty + 8 * slot, par ^ 1, abort_flag);
                                if (!ok) break;
                                // test hook (cp_selftest_stall): the tile is never loaded
                                if (P.stall == 8 /* CP_K_BWD_DQ */ && blockIdx.x == 0 && nload == 0) continue;
                                mbar_arrive_expect_tx(bar_kv_full + 8 * slot, Cfg::KTILE);
                                for (int h = 0; h < D / 64; ++h)
                                    tma_load_2d(sKV + slot * Cfg::KTILE + h * Cfg::KBOX,
                                                kv == 0 ? (const void*)&tmK : (const void*)&tmV, h * 64,
                                                kvrow, bar_kv_full + 8 * slot);
                            }
                        }
                    }
                }
            }
            if (!ok) {
                for (uint32_t n = (nload > Cfg::NSLOT ? nload - Cfg::NSLOT : 0); n < nload; ++n)
                    mbar_wait_drain(bar_kv_full + 8 * (n % Cfg::NSLOT), (n / Cfg::NSLOT) & 1);
                if (do_issued) mbar_wait_drain(bar_do_full, (iter & 1));
            }
        }
      } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // Order per key tile i: S(i) (once the elementwise warps have copied out
        // S(i-1)), dQ += dS(i-1) K(i-1) (dS sits in the dP columns), then dP(i)
        // over them (the tensor pipe runs in order).
        {
            constexpr uint32_t IDESC_S = idesc_bf16(128, Cfg::KT, false, false);
            constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);   // A tmem, B MN-major
            constexpr uint32_t KT16 = Cfg::KTILE >> 4;
            const uint32_t tS = tmem, tdP = tmem + 64, tQ = tmem + 128, tdQ = tmem + 256;
            const uint64_t dKV = sdesc_sw128(sKV, 16, 1024), dKVmn = sdesc_sw128(sKV, Cfg::KBOX, 1024);
            const uint64_t ddO = sdesc_sw128(sdO, 16, 1024);
            uint32_t nload = 0, iter = 0, sf_phase = 0, ae_phase = 0, p_phase = 0;
            bool ok = true, acc_busy = false, s_pending = false;
            // dQ += dS K for one finished key tile; dS of keys 16w .. +15 at dP columns 16w
            auto issue_dq = [&](uint32_t kslot, bool& first) -> bool {
                if (first && acc_busy) {   // every group has stored the previous item's dQ
                    if (!mbar_wait_warp(bar_acc_empty, ae_phase, abort_flag)) return false;
                    ae_phase ^= 1;
                    acc_busy = false;
                }
                if (!mbar_wait_warp(bar_p_full, p_phase, abort_flag)) return false;
                p_phase ^= 1;
                tc_fence_after();
                if (elect_one()) {
                    const uint64_t bk_mn = dKVmn + kslot * KT16;
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4)
                        mma_ts(tdQ, tdP + 16 * w4, bk_mn + ((w4 * 2048) >> 4), IDESC_G,
                               (!first || w4 > 0) ? 1u : 0u);
                    mma_commit(bar_kv_empty + 8 * kslot);
                }
                __syncwarp();
                first = false;
                return true;
            };
            for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
                const DqItem it = decode_dq<PD>(P, w);
                const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
                const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
                ok = mbar_wait_warp(bar_qt_full, iter & 1, abort_flag);   // Q rows in tensor memory
                if (!ok) break;
                ok = mbar_wait_warp(bar_do_full, iter & 1, abort_flag);   // dO tile in shared memory
                if (!ok) break;
                tc_fence_after();
                bool first = true, prev_live = false;
                uint32_t prev_kslot = 0;
                for (int s = P.s0; s < P.s1 && ok; ++s) {
                    const int j = __ldg(P.src + it.r * P.cp + s);
                    const KtSpan ks = kv_span<PD>(P, j, dsf, it.qo + 127 + P.nc, half);
                    for (int kt = kt_first(ks); kt < ks.b1 && ok; kt = kt_next(ks, kt)) {
                        const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                        for (int hh = 0; hh < 2 && ok; ++hh) {
                            if (classify_tile64(it.qo, dsf, dsl, ko128 + 64 * hh, P.nc) == TILE_SKIP) continue;
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
                            if (elect_one()) {
                                const uint64_t bk = dKV + kslot * KT16;
#pragma unroll
                                for (int k = 0; k < D / 16; ++k) {
                                    const uint32_t off = ((k / 4) * Cfg::KBOX + (k % 4) * 32) >> 4;
                                    mma_ts(tS, tQ + 8 * k, bk + off, IDESC_S, k > 0 ? 1u : 0u);
                                }
                                mma_commit(bar_st_ready);
                            }
                            __syncwarp();
                            s_pending = true;
                            // the previous tile's product reads dS from the dP columns ...
                            if (prev_live && !(ok = issue_dq(prev_kslot, first))) break;
                            // ... before this tile's dP overwrites them
                            ok = mbar_wait_warp(bar_kv_full + 8 * vslot, vpar, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                            if (elect_one()) {
                                const uint64_t bv = dKV + vslot * KT16;
#pragma unroll
                                for (int k = 0; k < D / 16; ++k) {
                                    const uint32_t offa = ((k / 4) * 16384 + (k % 4) * 32) >> 4;
                                    const uint32_t offb = ((k / 4) * Cfg::KBOX + (k % 4) * 32) >> 4;
                                    mma_ss(tdP, ddO + offa, bv + offb, IDESC_S, k > 0 ? 1u : 0u);
                                }
                                mma_commit(bar_dp_ready);
                                mma_commit(bar_kv_empty + 8 * vslot);
                            }
                            __syncwarp();
                            prev_live = true;
                            prev_kslot = kslot;
                        }
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
        const int wg = warp >> 2;                        // key columns [16wg, 16wg+16) of a tile
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + 16 * wg, tdP = tmem + lane_off + 64 + 16 * wg;
        const uint32_t tQ = tmem + lane_off + 128 + 32 * wg, tdQ = tmem + lane_off + 256 + 64 * wg;
        uint32_t st_phase = 0, dp_phase = 0, a_phase = 0, iter = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < P.n_items && ok; w += gridDim.x, ++iter) {
            const DqItem it = decode_dq<PD>(P, w);
            const int dsf = max(P.docs ? __ldg(P.doc_start + it.qpos) : 0, it.qo - P.wm1);
            const int dsl = max(P.docs ? __ldg(P.doc_start + it.qpos + 127) : 0, it.qo + 127 - P.wm1);
            const size_t rowi = static_cast<size_t>(it.bh) * P.q_rows + (it.qpos - P.q_base) + row;
            // this row's Q (bf16 pairs, elements [64wg, 64wg+64)) into tensor memory once the
            // previous item's S products have read the old one
            ok = __all_sync(0xffffffffu, mbar_wait(bar_qt_empty, (iter & 1) ^ 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            {
                const uint4* qsrc = reinterpret_cast<const uint4*>(P.q + rowi * D + 64 * wg);
                uint32_t qa[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = __ldg(qsrc + i);
                    qa[4 * i] = x.x; qa[4 * i + 1] = x.y; qa[4 * i + 2] = x.z; qa[4 * i + 3] = x.w;
                }
                tmem_st32(tQ, qa);
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
                    const int ko128 = tile_orig_of<PD>(P, j, kt, half);
                    for (int hh = 0; hh < 2 && ok; ++hh) {
                        const int ko = ko128 + 64 * hh;
                        const int cls = classify_tile64(it.qo, dsf, dsl, ko, P.nc);
                        if (cls == TILE_SKIP) continue;
                        // ---- S: copy out, release, and form P while dP is still being computed
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_st_ready, st_phase, abort_flag));
                        if (!ok) break;
                        st_phase ^= 1;
                        tc_fence_after();
                        const int lo = ds_q - ko - 16 * wg, hi = q_orig + P.nc - ko - 16 * wg;
                        float sv[16], dp[16];
                        tmem_ld16f(tS, sv);
                        tmem_wait_ld();
                        reg_fence16f(sv);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_s_free);   // the MMA warp may compute the next S
                        if (cls == TILE_FULL)
                            dq_p16<false>(sv, nlse2, P.scale_log2, 0, 0);
                        else
                            dq_p16<true>(sv, nlse2, P.scale_log2, lo, hi);
                        // ---- dP: copy out; the packed dS goes over this warp's own columns
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_ready, dp_phase, abort_flag));
                        if (!ok) break;
                        dp_phase ^= 1;
                        tc_fence_after();
                        tmem_ld16f(tdP, dp);
                        tmem_wait_ld();
                        reg_fence16f(dp);
                        uint32_t dk[8];
                        dq_ds16(sv, dp, dlt, dk);
                        tmem_st8(tdP, dk);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_full);
                        had = true;
                    }
                }
            }
            if (!ok) break;
            if (had) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_acc_full, a_phase, abort_flag));
                if (!ok) break;
                a_phase ^= 1;
                tc_fence_after();
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float a[32];
                    tmem_ld32f(tdQ + 32 * h, a);
                    tmem_wait_ld();
                    reg_fence32f(a);
                    if (P.dq32) {   // fp32 dQ, added into the caller's sum (this CTA owns the row)
                        float4* dq = reinterpret_cast<float4*>(P.dq32 + rowi * D + 64 * wg + 32 * h);
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
                        continue;
                    }
                    uint4* dq = reinterpret_cast<uint4*>(P.dq + rowi * D + 64 * wg + 32 * h);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dq[i] = make_uint4(pack_bf16(a[8 * i] * P.scale, a[8 * i + 1] * P.scale),
                                           pack_bf16(a[8 * i + 2] * P.scale, a[8 * i + 3] * P.scale),
                                           pack_bf16(a[8 * i + 4] * P.scale, a[8 * i + 5] * P.scale),
                                           pack_bf16(a[8 * i + 6] * P.scale, a[8 * i + 7] * P.scale));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty);
            } else if (!P.accumulate) {
                if (P.dq32) {
                    float4* dq = reinterpret_cast<float4*>(P.dq32 + rowi * D + 64 * wg);
                    for (int i = 0; i < 16; ++i) dq[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    uint4* dq = reinterpret_cast<uint4*>(P.dq + rowi * D + 64 * wg);
                    for (int i = 0; i < 8; ++i) dq[i] = make_uint4(0, 0, 0, 0);
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
