// Zigzag index maps.  Chunk c holds original tokens [c*C, (c+1)*C); virtual
// rank r holds chunk r then chunk 2cp-1-r, so shard position p = r*2C + t.
#pragma once

namespace cpattn {

// Original position of shard position p.
__host__ __device__ __forceinline__ int orig_of_shard(int p, int C, int cp)
{
    const int r = p / (2 * C), t = p - r * 2 * C;
    const int chunk = t < C ? r : 2 * cp - 1 - r;
    return chunk * C + (t < C ? t : t - C);
}

// Shard position of original position q.
__host__ __device__ __forceinline__ int shard_of_orig(int q, int C, int cp)
{
    const int c = q / C, t = q - c * C;
    return c < cp ? c * 2 * C + t : (2 * cp - 1 - c) * 2 * C + C + t;
}

}  // namespace cpattn
