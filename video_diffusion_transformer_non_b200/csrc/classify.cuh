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

// 3D neighbourhood windows (vidattn_fwd_window): for every (b, 128-token
// tile) of coord_q and coord_kv, the bounding box of the tile's (t, h, w)
// coordinates, int4 {t_lo | t_hi << 16, h_lo | h_hi << 16, w_lo | w_hi << 16,
// raster} (coordinates packed per token as t << 22 | h << 11 | w).  The
// attention kernel skips a key tile whose box misses the union of its
// queries' windows and takes the unmasked path where the box lies inside
// every query's window.  raster = 1 when every token x of the tile sits at
// the raster position of its index in a volume of rows of Wg tokens (t = x /
// (Hg Wg), h = x / Wg mod Hg, w = x mod Wg) and Wg >= kRasterMinW: the
// kernel then builds a row's mask from the tile index alone.  Launch shape
// as seg_tile_classify_kernel.
constexpr int kRasterMinW = 10;   // at most 16 (t, h) rows in a 128-key tile
__global__ void __launch_bounds__(128) win_tile_bbox_kernel(
    const int32_t* __restrict__ coord_q, const int32_t* __restrict__ coord_kv,
    int4* __restrict__ q_box, int4* __restrict__ kv_box, int S_q, int S_kv, int T, int Hg,
    int Wg) {
  const int which = blockIdx.z;
  const int b = blockIdx.y;
  const int tile = blockIdx.x;
  const int S = which ? S_kv : S_q;
  const int n_tiles = (S + kSegTile - 1) / kSegTile;
  if (tile >= n_tiles) return;
  const int32_t* coord = (which ? coord_kv : coord_q) + static_cast<int64_t>(b) * S;
  const int idx = tile * kSegTile + threadIdx.x;
  int lo[3] = {INT_MAX, INT_MAX, INT_MAX}, hi[3] = {INT_MIN, INT_MIN, INT_MIN};
  bool raster = Wg >= kRasterMinW;
  if (idx < S) {
    const uint32_t c = static_cast<uint32_t>(__ldg(coord + idx));
    lo[0] = hi[0] = int(c >> 22);
    lo[1] = hi[1] = int((c >> 11) & 2047u);
    lo[2] = hi[2] = int(c & 2047u);
    const int row = idx / Wg;
    raster = raster && row / Hg < T &&
             c == (uint32_t(row / Hg) << 22 | uint32_t(row % Hg) << 11 | uint32_t(idx % Wg));
  }
  raster = __syncthreads_and(raster) != 0;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo[a] = min(lo[a], __shfl_xor_sync(0xffffffffu, lo[a], o));
      hi[a] = max(hi[a], __shfl_xor_sync(0xffffffffu, hi[a], o));
    }
  }
  __shared__ int s_lo[3][4], s_hi[3][4];
  const int warp = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      s_lo[a][warp] = lo[a];
      s_hi[a][warp] = hi[a];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int packed[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const int l = min(min(s_lo[a][0], s_lo[a][1]), min(s_lo[a][2], s_lo[a][3]));
      const int h = max(max(s_hi[a][0], s_hi[a][1]), max(s_hi[a][2], s_hi[a][3]));
      packed[a] = l | (h << 16);
    }
    int4* dst = (which ? kv_box : q_box) + static_cast<int64_t>(b) * n_tiles + tile;
    *dst = make_int4(packed[0], packed[1], packed[2], raster ? 1 : 0);
  }
}

}  // namespace vidattn
