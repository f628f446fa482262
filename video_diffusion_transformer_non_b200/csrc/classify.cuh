// Segment-id tile summaries: for every (b, 128-token tile) of seg_q and seg_kv,
// {min id, max id, uniform flag}.  The attention kernel derives the class of a
// (query tile, key tile) pair from two summaries: "skip" when the id ranges
// are disjoint (no query can see any key: the tile is never loaded), "full"
// when both tiles hold one and the same id (no per-element mask), otherwise
// "mixed" (per-element mask).  This is how key blocks with no valid pair are
// skipped without building a dense mask (vidax: A Unified JAX Framework for
// Video Generative Models on Accelerator Meshes, Appendix A, Table 4, group 2,
// row "HunyuanVideo-1.5: RESOURCE_EXHAUSTED at 720p").
#pragma once
#include <climits>
#include <cstdint>

namespace vidattn {

constexpr int kSegTile = 128;

// grid (max(n_q_tiles, n_kv_tiles), B, 2), block 128.  z = 0: seg_q -> q_sum,
// z = 1: seg_kv -> kv_sum.  Summaries are int4 {min, max, uniform, 0} stored
// [B][n_tiles]; the ragged last tile summarises its valid tokens only.
__global__ void __launch_bounds__(128) seg_tile_classify_kernel(
    const int32_t* __restrict__ seg_q, const int32_t* __restrict__ seg_kv,
    int4* __restrict__ q_sum, int4* __restrict__ kv_sum, int S_q, int S_kv) {
  const int which = blockIdx.z;
  const int b = blockIdx.y;
  const int tile = blockIdx.x;
  const int S = which ? S_kv : S_q;
  const int n_tiles = (S + kSegTile - 1) / kSegTile;
  if (tile >= n_tiles) return;
  const int32_t* seg = (which ? seg_kv : seg_q) + static_cast<int64_t>(b) * S;
  const int idx = tile * kSegTile + threadIdx.x;
  int lo = INT_MAX, hi = INT_MIN;
  if (idx < S) lo = hi = __ldg(seg + idx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  __shared__ int s_lo[4], s_hi[4];
  const int warp = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) { s_lo[warp] = lo; s_hi[warp] = hi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    lo = min(min(s_lo[0], s_lo[1]), min(s_lo[2], s_lo[3]));
    hi = max(max(s_hi[0], s_hi[1]), max(s_hi[2], s_hi[3]));
    int4* dst = (which ? kv_sum : q_sum) + static_cast<int64_t>(b) * n_tiles + tile;
    *dst = make_int4(lo, hi, lo == hi ? 1 : 0, 0);
  }
}

}  // namespace vidattn
