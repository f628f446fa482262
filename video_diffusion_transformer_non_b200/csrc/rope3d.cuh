// 3D rotary position embedding of q and k, one memory-bound pass.
//
// vidax (§2, "3D RoPE, 3D VAEs, and flash attention") rotates q and k over the
// time, height and width axes of the video latent before attention and gives
// no formula; the rotation here is RoFormer's (Su et al. 2021), applied per
// axis: the head dim is cut into a t band, an h band and a w band, feature
// pair k of a band of d features turns by coord * theta^(-2k/d), and tokens
// outside the video range are copied unchanged.  include/vidattn.h
// (vidattn_rope3d) states the argument contract.
//
// Work split: a tile is kRopeTokens consecutive tokens of every (tensor, b, h)
// slab.  The CTA computes the tile's (cos, sin) table once in shared memory
// (the angles in fp64, reduced to [-pi, pi], then sincosf; two tables
// alternate, so one barrier per tile suffices), each thread keeps the entries
// of its own 8 features in registers and then streams 16-byte chunks of all
// slabs through them: 8 loads in flight per thread (4 with the half-split
// pairing, whose staging needs more registers), streaming-cache loads and
// stores (every byte is touched once).  The
// interleaved pairing finds both features of a pair in one chunk; the
// half-split pairing stages the chunk in shared memory and reads the partner
// feature from the neighbouring thread of the same row.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace vidattn {

constexpr int kRopeThreads = 256;
constexpr int kRopeTokens = 8;
constexpr int kRopeMaxD = 128;

struct RopeParams {
  const uint16_t* in[2];
  uint16_t* out[2];
  long long sb, sh, ss;        // input strides in elements (batch, head, token)
  int n_slabs;                 // n_tensors * B * H
  int S;
  FastDiv div_bh, div_h;       // by B * H and by H
  int n_video, hw, Hg, Wg, offset;
  int col_h, col_w;            // first table column of the h band and of the w band
  double freq[kRopeMaxD / 2];  // per table column: theta^(-2k/d)
  // per feature e: its table column, its partner feature, and 1 when e is the
  // first feature of its pair (its partner's term enters with a minus sign)
  uint8_t col[kRopeMaxD], partner[kRopeMaxD], first[kRopeMaxD];
};

__device__ __forceinline__ uint4 ld_stream_v4(const uint16_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream_v4(uint16_t* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int D, bool kInterleaved>
__global__ void __launch_bounds__(kRopeThreads) rope3d_kernel(const __grid_constant__ RopeParams p) {
  constexpr int kHalf = D / 2;
  constexpr int kChunks = D / 8;                           // 16-byte chunks per row
  constexpr int kPerSlab = kRopeTokens * kChunks;          // threads per slab
  constexpr int kSlabsPerPass = kRopeThreads / kPerSlab;
  static_assert(kRopeThreads % kPerSlab == 0 && 32 % kChunks == 0, "tile shape");
  constexpr int kRopeUnroll = kInterleaved ? 8 : 4;   // 16-byte loads in flight per thread

  __shared__ __align__(16) float2 table[2][kRopeTokens][kHalf];
  __shared__ uint4 stage[kInterleaved ? 1 : kRopeUnroll][kRopeThreads];

  const int tid = threadIdx.x;
  const int ch = tid % kChunks;
  const int row = (tid / kChunks) % kRopeTokens;
  const int slab_lane = tid / kPerSlab;
  const int n_tiles = (p.S + kRopeTokens - 1) / kRopeTokens;

  // this thread's features: table columns, and for the half-split pairing
  // the partner's position in the staged row
  int col[8], partner_chunk[8], partner_elem[8];
  bool first[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int f = ch * 8 + e;
    col[e] = p.col[f];
    first[e] = p.first[f] != 0;
    partner_chunk[e] = p.partner[f] / 8;
    partner_elem[e] = p.partner[f] % 8;
  }

  int parity = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, parity ^= 1) {
    const int s0 = tile * kRopeTokens;
    // this tile's table goes to the buffer read two tiles ago: every thread
    // has passed the previous tile's barrier, so it is done reading it
    float2 (*tb)[kHalf] = table[parity];
    for (int i = tid; i < kRopeTokens * kHalf; i += kRopeThreads) {
      const int r = i / kHalf, c = i % kHalf;
      const int n = s0 + r - p.offset;
      float cv = 1.f, sv = 0.f;
      if (n >= 0 && n < p.n_video) {
        const int coord = c < p.col_h ? n / p.hw : (c < p.col_w ? (n / p.Wg) % p.Hg : n % p.Wg);
        const double two_pi = 6.283185307179586476925286766559;
        double a = double(coord) * p.freq[c];
        a -= two_pi * rint(a / two_pi);
        sincosf(float(a), &sv, &cv);
      }
      tb[r][c] = make_float2(cv, sv);
    }
    __syncthreads();

    float cs[8], sn[8];
    if constexpr (kInterleaved) {
      // features 8ch .. 8ch+7 are the pairs (columns) 4ch .. 4ch+3
      const float4 a = *reinterpret_cast<const float4*>(&tb[row][4 * ch]);
      const float4 b = *reinterpret_cast<const float4*>(&tb[row][4 * ch + 2]);
      const float cc[4] = {a.x, a.z, b.x, b.z}, ss[4] = {a.y, a.w, b.y, b.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cs[e] = cc[e >> 1];
        sn[e] = (e & 1) ? ss[e >> 1] : -ss[e >> 1];
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 t = tb[row][col[e]];
        cs[e] = t.x;
        sn[e] = first[e] ? -t.y : t.y;
      }
    }
    const int s = s0 + row;
    const bool row_ok = s < p.S;

    for (int base = slab_lane; base < p.n_slabs; base += kSlabsPerPass * kRopeUnroll) {
      uint4 v[kRopeUnroll];
      uint16_t* dst[kRopeUnroll];
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const int slab = base + u * kSlabsPerPass;
        v[u] = make_uint4(0, 0, 0, 0);
        dst[u] = nullptr;
        if (row_ok && slab < p.n_slabs) {
          const uint32_t t = fastdiv(uint32_t(slab), p.div_bh);
          const uint32_t bh = uint32_t(slab) - t * p.div_bh.d;
          const uint32_t b = fastdiv(bh, p.div_h);
          const uint32_t h = bh - b * p.div_h.d;
          const uint16_t* src = p.in[t] + b * p.sb + h * p.sh + s * p.ss + ch * 8;
          dst[u] = p.out[t] + (static_cast<long long>(bh) * p.S + s) * D + ch * 8;
          v[u] = ld_stream_v4(src);
        }
      }
      if constexpr (!kInterleaved) {
#pragma unroll
        for (int u = 0; u < kRopeUnroll; ++u) stage[u][tid] = v[u];
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        float x[8], y[8], xp[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x[2 * j] = bf16_lo(w[j]);
          x[2 * j + 1] = bf16_hi(w[j]);
        }
        if constexpr (kInterleaved) {
#pragma unroll
          for (int e = 0; e < 8; ++e) xp[e] = x[e ^ 1];
        } else {
          const uint16_t* rowbase =
              reinterpret_cast<const uint16_t*>(&stage[u][tid - ch]);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            xp[e] = __uint_as_float(uint32_t(rowbase[partner_chunk[e] * 8 + partner_elem[e]]) << 16);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = fmaf(x[e], cs[e], xp[e] * sn[e]);
        if (dst[u] != nullptr) {
          uint4 o;
          o.x = pack_bf16x2(y[0], y[1]);
          o.y = pack_bf16x2(y[2], y[3]);
          o.z = pack_bf16x2(y[4], y[5]);
          o.w = pack_bf16x2(y[6], y[7]);
          st_stream_v4(dst[u], o);
        }
      }
      if constexpr (!kInterleaved) __syncwarp();
    }
  }
}

}  // namespace vidattn
