// LSE merge: combine n partial attentions of the same query rows into the
// attention over the union of their key sets (the concept guide's
// "combine(attn)" step, read as the exact log-sum-exp merge).
//
// For a row with partials (O_i, L_i):  m = max_i L_i,  w_i = exp(L_i - m)
// (0 for L_i = -inf), L = m + ln sum_i w_i, O = sum_i w_i O_i / sum_i w_i.
// This is the closed form of folding the partials pairwise in order; a row
// whose partials are all -inf stays (0, -inf).
//
// HBM-bound: each warp owns one row at a time; lane l reads columns
// [4l, 4l+4) (and [128+4l, ...) for head_dim > 128) of each live partial with
// 16-byte loads, so a warp reads 512 contiguous bytes per partial.  Partials
// with L = -inf are not read.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace cpattn {

constexpr int MERGE_MAX_PARTS = 64;

struct MergeParams {
    int64_t rows;
    int32_t D, n_parts;
    const float* o_parts;    // [n][rows][D]
    const float* lse_parts;  // [n][rows]
    __nv_bfloat16* o_out;    // [rows][D]
    float* lse_out;          // [rows]
};

__global__ void __launch_bounds__(256) lse_merge_kernel(MergeParams M)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int nvec = M.D / 4;            // float4 per row
    const bool two = nvec > 32;          // head_dim > 128: two vectors per lane
    for (int64_t row = warp_g; row < M.rows; row += nwarps) {
        // lane p holds L of parts p and p+32
        float la = lane < M.n_parts ? __ldg(M.lse_parts + static_cast<int64_t>(lane) * M.rows + row) : -INFINITY;
        float lb = lane + 32 < M.n_parts ? __ldg(M.lse_parts + static_cast<int64_t>(lane + 32) * M.rows + row) : -INFINITY;
        float m = fmaxf(la, lb);
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
        float wsum = 0.f;
        if (m != -INFINITY) {
            const float wa = la == -INFINITY ? 0.f : expf(la - m);
            const float wb = lb == -INFINITY ? 0.f : expf(lb - m);
            float ws = wa + wb;
            for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
            wsum = ws;
            for (int p = 0; p < M.n_parts; ++p) {
                const float w = __shfl_sync(0xffffffffu, p < 32 ? wa : wb, p & 31);
                if (w == 0.f) continue;  // warp-uniform
                const float4* src = reinterpret_cast<const float4*>(
                    M.o_parts + (static_cast<int64_t>(p) * M.rows + row) * M.D);
                if (lane < nvec) {
                    const float4 x = __ldg(src + lane);
                    acc0.x += w * x.x; acc0.y += w * x.y; acc0.z += w * x.z; acc0.w += w * x.w;
                }
                if (two && lane + 32 < nvec) {
                    const float4 x = __ldg(src + lane + 32);
                    acc1.x += w * x.x; acc1.y += w * x.y; acc1.z += w * x.z; acc1.w += w * x.w;
                }
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        uint2* dst = reinterpret_cast<uint2*>(M.o_out + row * M.D);
        if (lane < nvec)
            dst[lane] = make_uint2(pack_bf16(acc0.x * inv, acc0.y * inv), pack_bf16(acc0.z * inv, acc0.w * inv));
        if (two && lane + 32 < nvec)
            dst[lane + 32] = make_uint2(pack_bf16(acc1.x * inv, acc1.y * inv), pack_bf16(acc1.z * inv, acc1.w * inv));
        if (lane == 0) M.lse_out[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
    }
}

// The same merge over partials in the forward's tile-interleaved layout: for
// part p, 128-row tile t (rows 128t .. 128t+127 of the part), column group c4 (4
// floats) and row r of the tile, the float4 at ((p * ntile + t) * D/4 + c4) * 128 + r.
// The forward writes this layout for its own workspace because a warp's 32
// rows then store 512 contiguous bytes per instruction (row-major partials
// would put each lane of every store in a different line).  One CTA of 256
// threads per tile, two threads per row (each half of the column groups): the
// weights go to shared memory, the loads of each (part, column group) are 512
// contiguous bytes per warp, and the tile's bf16 output is staged in shared
// memory (rows padded by 8 bytes) and written back as one contiguous block.
__global__ void __launch_bounds__(256) lse_merge_tiled_kernel(MergeParams M)
{
    extern __shared__ float msm[];
    const int r = threadIdx.x & 127, hh = threadIdx.x >> 7;
    const int nvec = M.D / 4;
    const int64_t ntile = M.rows / 128;
    float* w_s = msm;                                                  // [n_parts][128]
    float* inv_s = msm + M.n_parts * 128;                              // [128]
    uint2* o_s = reinterpret_cast<uint2*>(msm + M.n_parts * 128 + 128);   // [128][nvec + 1]
    const float4* parts = reinterpret_cast<const float4*>(M.o_parts);
    for (int64_t t = blockIdx.x; t < ntile; t += gridDim.x) {
        const int64_t row = t * 128 + r;
        if (hh == 0) {
            float m = -INFINITY;
            for (int p = 0; p < M.n_parts; ++p) {
                const float l = __ldg(M.lse_parts + static_cast<int64_t>(p) * M.rows + row);
                w_s[p * 128 + r] = l;
                m = fmaxf(m, l);
            }
            for (int p = 0; p < M.n_parts; ++p) {
                const float l = w_s[p * 128 + r];
                w_s[p * 128 + r] = (m == -INFINITY || l == -INFINITY) ? 0.f : expf(l - m);
            }
            // sum of the weights in the order of lse_merge_kernel's warp reduction (part
            // pairs p, p+32, then a butterfly over the 32 lanes), folded in place, so the
            // two kernels give the same bits for the same partials
            float v[32];
#pragma unroll
            for (int l = 0; l < 32; ++l)
                v[l] = (l < M.n_parts ? w_s[l * 128 + r] : 0.f) +
                       (l + 32 < M.n_parts ? w_s[(l + 32) * 128 + r] : 0.f);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int l = 0; l < off; ++l) v[l] = v[l] + v[l + off];
            const float wsum = m == -INFINITY ? 0.f : v[0];
            inv_s[r] = wsum > 0.f ? 1.f / wsum : 0.f;
            M.lse_out[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
        }
        __syncthreads();
        const float inv = inv_s[r];
        // this thread's half of the column groups, four at a time: four independent
        // 16-byte loads per live part
        for (int c0 = hh * (nvec / 2); c0 < (hh + 1) * (nvec / 2); c0 += 4) {
            float4 acc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            // dead parts (weight 0: never written) are not loaded and add nothing; the
            // loads are predicated rather than branched around so that those of
            // several parts are in flight together
#pragma unroll 4
            for (int p = 0; p < M.n_parts; ++p) {
                const float w = w_s[p * 128 + r];
                const float4* src = parts + ((static_cast<int64_t>(p) * ntile + t) * nvec + c0) * 128 + r;
                float4 x[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    x[j] = w != 0.f ? __ldg(src + j * 128) : make_float4(0.f, 0.f, 0.f, 0.f);
                if (w != 0.f) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[j].x += w * x[j].x; acc[j].y += w * x[j].y;
                        acc[j].z += w * x[j].z; acc[j].w += w * x[j].w;
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o_s[r * (nvec + 1) + c0 + j] = make_uint2(pack_bf16(acc[j].x * inv, acc[j].y * inv),
                                                          pack_bf16(acc[j].z * inv, acc[j].w * inv));
        }
        __syncthreads();
        // the tile's 128 output rows are contiguous: 8-byte stores, 256 contiguous bytes per warp
        uint2* dst = reinterpret_cast<uint2*>(M.o_out + t * 128 * M.D);
        for (int i = threadIdx.x; i < 128 * nvec; i += 256) {
            const int rr = i / nvec, cc = i - rr * nvec;
            dst[i] = o_s[rr * (nvec + 1) + cc];
        }
        __syncthreads();
    }
}

}  // namespace cpattn
