// Shard planner / indexer and the shard gather.
//
// The sequence of S tokens is cut into 2*cp chunks of C = S/(2cp) tokens
// (S % (2*cp) == 0: NeMo "Hierarchical Context Parallel Skill", "Required
// constraints"); virtual rank r owns chunk r followed by chunk 2cp-1-r, so a
// rank's early (cheap) causal rows are paired with late (expensive) ones and
// every rank gets the same causal work.  K/V shards are visited in all-gather
// order (s) or ring order ((r - s) mod cp) (Accelerate "Context Parallel"
// concept guide, "all-to-all vs all-gather").
//
// All outputs are integers and bit-exact.
#pragma once
#include "ptx.cuh"
#include "zigzag.cuh"

namespace cpattn {

constexpr int PLAN_MAX_CP = 1024;

struct PlanParams {
    int32_t S, cp, C, num_docs, docs, rotate;
    int32_t wm1;        // sliding window - 1 (larger than S: no window)
    int32_t causal;     // 0: every query sees every key (no causal mask, no documents)
    int32_t per_doc;    // 1: every document cut into 2cp chunks (FlashCP Per-Doc sharding)
    const int32_t* cu;  // [num_docs+1] original order (docs only)
    int32_t *perm, *inv_perm, *src, *doc_start, *rank_cu_off, *rank_cu;
    int32_t *tile_orig, *tile_shard;   // [S/128] each
    int64_t* pairs;
};

// Per-document sharding: the shard position of original position o, whose
// document starts at s and has length L = 2cp * c.  o sits in chunk i = (o - s) / c
// at offset w; rank r = i (i < cp) or 2cp-1-i holds, document after document, its
// chunk r then its chunk 2cp-1-r, so the documents before o's fill s / cp of its
// local rows.
__device__ __forceinline__ int per_doc_shard_pos(int o, int s, int c, int C, int cp)
{
    const int i = (o - s) / c, w = (o - s) - i * c;
    const int r = i < cp ? i : 2 * cp - 1 - i;
    return r * 2 * C + s / cp + (i < cp ? 0 : c) + w;
}

// Largest d in [0, nd-1] with cu[d] <= x (cu[0] = 0 <= x for a valid list).
__device__ __forceinline__ int doc_index(const int32_t* cu, int nd, int x)
{
    int lo = 0, hi = nd - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Number of document starts strictly inside (a, a + len) (cu[1..nd-1]).
__device__ __forceinline__ int doc_starts_inside(const int32_t* cu, int nd, int a, int len)
{
    if (nd <= 1) return 0;
    int d = doc_index(cu, nd, a) + 1;  // first start > a (if cu valid)
    int n = 0;
    while (d < nd && __ldg(cu + d) < a + len) {
        if (__ldg(cu + d) > a) ++n;
        ++d;
    }
    return n;
}

// One block: validate cu_seqlens, zero the pair counters, write src and the
// per-rank local segment lists.
__global__ void __launch_bounds__(256) plan_meta_kernel(PlanParams P)
{
    __shared__ int32_t cnt[PLAN_MAX_CP + 1];
    const int tid = threadIdx.x;
    if (P.docs) {
        bool bad = false, uneven = false;
        if (tid == 0) bad = (__ldg(P.cu) != 0) || (__ldg(P.cu + P.num_docs) != P.S);
        for (int d = tid; d < P.num_docs; d += blockDim.x) {
            const int len = __ldg(P.cu + d + 1) - __ldg(P.cu + d);
            if (len <= 0) bad = true;
            // per-document chunks must be whole 128-row tiles for the attention kernels
            if (P.per_doc && len % (256 * P.cp) != 0) uneven = true;
        }
        if (bad) record_status(1 /* CP_ERR_INVALID_ARG */);
        else if (uneven) record_status(2 /* CP_ERR_UNSUPPORTED */);
    }
    if (P.per_doc) {
        // every map starts as the identity, so whatever the document list, every
        // index a later kernel reads from the plan stays inside the sequence
        for (int p = tid; p < P.S; p += blockDim.x) {
            P.perm[p] = p;
            P.inv_perm[p] = p;
        }
        for (int t = tid; t < P.S / 128; t += blockDim.x) {
            P.tile_orig[t] = t * 128;
            P.tile_shard[t] = t;
        }
    }
    for (int i = tid; i < P.cp * P.cp; i += blockDim.x) {
        const int r = i / P.cp, s = i - r * P.cp;
        P.src[i] = P.rotate == 0 ? s : ((r - s) % P.cp + P.cp) % P.cp;
    }
    for (int r = tid; r < P.cp; r += blockDim.x) {
        P.pairs[r] = 0;
        int n = 3;  // local 0, chunk boundary C, end 2C
        if (P.per_doc) {
            n = 2 * P.num_docs + 1;  // each document's two chunks, then 2C
        } else if (P.docs) {
            n += doc_starts_inside(P.cu, P.num_docs, r * P.C, P.C);
            n += doc_starts_inside(P.cu, P.num_docs, (2 * P.cp - 1 - r) * P.C, P.C);
        }
        cnt[r] = n;
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int r = 0; r < P.cp; ++r) {
            const int n = cnt[r];
            cnt[r] = acc;
            P.rank_cu_off[r] = acc;
            acc += n;
        }
        P.rank_cu_off[P.cp] = acc;
    }
    __syncthreads();
    for (int r = tid; r < P.cp && P.per_doc; r += blockDim.x) {
        int w = cnt[r];
        for (int d = 0; d < P.num_docs; ++d) {
            const int s0 = __ldg(P.cu + d), c = (__ldg(P.cu + d + 1) - s0) / (2 * P.cp);
            P.rank_cu[w++] = s0 / P.cp;
            P.rank_cu[w++] = s0 / P.cp + c;
        }
        P.rank_cu[w++] = 2 * P.C;
    }
    for (int r = tid; r < P.cp && !P.per_doc; r += blockDim.x) {
        int w = cnt[r];
        for (int half = 0; half < 2; ++half) {
            const int chunk = half == 0 ? r : 2 * P.cp - 1 - r;
            const int a = chunk * P.C;
            P.rank_cu[w++] = half * P.C;
            if (P.docs && P.num_docs > 1) {
                int d = doc_index(P.cu, P.num_docs, a) + 1;
                while (d < P.num_docs && __ldg(P.cu + d) < a + P.C) {
                    const int x = __ldg(P.cu + d);
                    if (x > a) P.rank_cu[w++] = half * P.C + (x - a);
                    ++d;
                }
            }
        }
        P.rank_cu[w++] = 2 * P.C;
    }
}

// Grid over shard positions: perm, inv_perm, doc_start and the per-rank
// unmasked pair counts (keys max(doc_start(o), o - wm1) .. o for the token at
// original o under the causal mask; all S keys without it).
__global__ void __launch_bounds__(256) plan_index_kernel(PlanParams P)
{
    const int n2c = 2 * P.C;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x; base < P.S;
         base += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int p = static_cast<int>(base) + threadIdx.x;
        int64_t cnt = 0;
        int r = -1;
        if (p < P.S && !P.per_doc) {
            r = p / n2c;
            const int t = p - r * n2c;
            const int chunk = t < P.C ? r : 2 * P.cp - 1 - r;
            const int o = chunk * P.C + (t < P.C ? t : t - P.C);
            P.perm[p] = o;
            P.inv_perm[o] = p;
            if ((p & 127) == 0) {
                P.tile_orig[p >> 7] = o;
                P.tile_shard[o >> 7] = p >> 7;
            }
            const int ds = P.docs ? __ldg(P.cu + doc_index(P.cu, P.num_docs, o)) : 0;
            P.doc_start[p] = ds;
            cnt = P.causal ? static_cast<int64_t>(min(o - ds, P.wm1)) + 1 : static_cast<int64_t>(P.S);
        } else if (p < P.S) {
            // per-document sharding: this thread takes ORIGINAL position o = p
            const int o = p;
            const int d = doc_index(P.cu, P.num_docs, o);
            const int s0 = __ldg(P.cu + d), len = __ldg(P.cu + d + 1) - s0;
            // a document the list does not describe validly keeps the identity (the
            // status word says why); the checks keep every index inside [0, S)
            int q = o;
            if (len > 0 && len % (256 * P.cp) == 0 && s0 >= 0 && s0 % (256 * P.cp) == 0 && s0 <= o &&
                o - s0 < len && len <= P.S - s0)
                q = per_doc_shard_pos(o, s0, len / (2 * P.cp), P.C, P.cp);
            P.perm[q] = o;
            P.inv_perm[o] = q;
            if ((o & 127) == 0) {
                P.tile_orig[q >> 7] = o;
                P.tile_shard[o >> 7] = q >> 7;
            }
            P.doc_start[q] = s0;
            r = q / n2c;
            cnt = static_cast<int64_t>(min(o - s0, P.wm1)) + 1;
        }
        // warp-level sum when the whole warp belongs to one rank, else per thread
        const int r0 = __shfl_sync(0xffffffffu, r, 0), r31 = __shfl_sync(0xffffffffu, r, 31);
        if (r0 == r31 && r0 >= 0) {
            for (int off = 16; off > 0; off >>= 1)
                cnt += __shfl_down_sync(0xffffffffu, cnt, off);
            if ((threadIdx.x & 31) == 0)
                atomicAdd(reinterpret_cast<unsigned long long*>(P.pairs + r0),
                          static_cast<unsigned long long>(cnt));
        } else if (r >= 0) {
            atomicAdd(reinterpret_cast<unsigned long long*>(P.pairs + r),
                      static_cast<unsigned long long>(cnt));
        }
    }
}

// Row gather between original and shard order for one tensor
// [outer][S][row_bytes] (row_bytes a multiple of 16).  to_shard = 1:
// out[o][p] = in[o][orig(p)]; to_shard = 0: out[o][q] = in[o][shard(q)].
struct GatherParams {
    const uint4* in;
    uint4* out;
    int64_t rows;       // outer * S
    int32_t vpr;        // 16-byte vectors per row
    int32_t rpw;        // rows per warp pass (32 / vpr when vpr divides 32, else 1)
    int32_t S, C, cp, to_shard;
    const int32_t* map;   // per-document plans: perm (to shard) or inv_perm (back); else null
};

template <bool MAP>
__global__ void __launch_bounds__(256) gather_rows_kernel(GatherParams G)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int sub = G.rpw > 1 ? lane / G.vpr : 0;
    const int e0 = G.rpw > 1 ? lane - sub * G.vpr : lane;
    constexpr int U = 4;
    for (int64_t rb = warp_g * G.rpw * U; rb < G.rows; rb += nwarps * G.rpw * U) {
        uint4 buf[U][1];
        int64_t dst_row[U];
        bool valid[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = rb + static_cast<int64_t>(u) * G.rpw + sub;
            valid[u] = row < G.rows;
            dst_row[u] = row;
            if (valid[u]) {
                const int64_t o = row / G.S;
                const int p = static_cast<int>(row - o * G.S);
                const int sp = MAP ? __ldg(G.map + p)
                                     : (G.to_shard ? orig_of_shard(p, G.C, G.cp) : shard_of_orig(p, G.C, G.cp));
                const int64_t srow = o * G.S + sp;
                if (e0 < G.vpr) buf[u][0] = __ldg(G.in + srow * G.vpr + e0);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (valid[u] && e0 < G.vpr) G.out[dst_row[u] * G.vpr + e0] = buf[u][0];
        // rows wider than 32 vectors: remaining vectors of the same rows
        if (G.rpw == 1 && G.vpr > 32) {
            for (int e = e0 + 32; e < G.vpr; e += 32) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!valid[u]) continue;
                    const int64_t row = dst_row[u];
                    const int64_t o = row / G.S;
                    const int p = static_cast<int>(row - o * G.S);
                    const int sp = MAP ? __ldg(G.map + p)
                                         : (G.to_shard ? orig_of_shard(p, G.C, G.cp) : shard_of_orig(p, G.C, G.cp));
                    G.out[row * G.vpr + e] = __ldg(G.in + (o * G.S + sp) * G.vpr + e);
                }
            }
        }
    }
}

}  // namespace cpattn
