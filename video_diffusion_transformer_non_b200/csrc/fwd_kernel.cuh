// Masked multi-head attention forward for sm_100a.
//
// Computes, per (b, h, query row i), softmax over the keys j visible to the
// query of scale * q_i . k_j, applied to v, plus the natural log-sum-exp of
// the visible scaled logits.  A key is visible when the segment ids match
// (every key when no ids are given), and, with the options, when it lies
// within the causal limit j <= i + (S_kv - S_q) or in the query's 3D
// neighbourhood window.  The full query-key matrix is never stored: scores
// live only in tensor memory one 128x128 tile at a time and an online softmax
// carries the running offset and sum (vidax: A Unified JAX Framework for
// Video Generative Models on Accelerator Meshes, §2 "3D RoPE, 3D VAEs, and
// flash attention", which dispatches such attention to flash-attention
// kernels, its reference [2]); key tiles that no query of the CTA can see are
// skipped, not masked (same paper, Appendix A, Table 4, group 2, row
// "HunyuanVideo-1.5: RESOURCE_EXHAUSTED at 720p").
//
// Work unit = (b, h, 256 query rows as two 128-row tiles Q0, Q1[, one of
// n_split ranges of the key tiles]).  One CTA per unit, or a persistent grid
// of one CTA per SM, each CTA looping over units with every barrier phase
// running on.  384 threads:
//   warps 0-3  softmax for Q0 (TMEM lanes 0-127 = the tile's rows), epilogue
//   warps 4-7  softmax for Q1, epilogue
//   warp  8    allocates TMEM; runs the tensor-core schedule converged, an
//              elected lane issuing every tcgen05.mma and commit
//   warp  9    runs the load schedule converged, an elected lane issuing
//              every TMA load (Q0, Q1 once per unit; then K_j, V_j)
//   warp  10   with ids or windows: lists each unit's visited key tiles
//   warp  11   idle
// Tensor memory (512 columns x 128 lanes, fp32), D = 128:
//   [0,128) S0 / P0   [128,256) S1 / P1   [256,384) O0   [384,512) O1
// P (bf16, two per column) overwrites the first 64 columns of its S tile.
// D = 64 (kSepP): S0, S1 in [0,256), P0, P1 in [256,384), O0, O1 in [384,512);
// the softmax moves its S row into registers and releases S once P is
// computed (the exponentials consume the S registers as they go).
// Shared memory: Q0, Q1, then a ring of kStages K-or-V tiles; every tile is
// [D/64][128 rows][64 columns] bf16 written by TMA with 128-byte swizzle.
//
// Tensor-core order for D = 128 (in issue order; each tile pair t):
//   S0 = Q0 K_0^T, S1 = Q1 K_0^T, then for t = 0..n-1:
//   O0 += P0 V_t, S0 = Q0 K_{t+1}^T, O1 += P1 V_t, S1 = Q1 K_{t+1}^T
// so the tensor core works on one Q tile while the other's softmax runs.
// The softmax uses a running offset: after a row's first tile P = 2^(c s - m)
// with the row's previous offset m and no tile maximum; only a tile whose sum
// of P exceeds 2^32, a masked tile (except in the kMaskFast variant), a row's
// first tile or scale <= 0 takes the exact path (tile maximum; O and the row
// sum rescaled when the maximum grows by more than 2^8).  A masked tile's key
// ids or coordinates are staged per warp in shared memory and each row builds
// a 128-bit mask from them.
#pragma once
#include <climits>
#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"

namespace vidattn {

constexpr int kBM = 128;        // query rows per Q tile
constexpr int kBN = 128;        // keys per K/V tile
constexpr int kFwdThreads = 384;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kStaleSumLimit = 4294967296.0f;   // 2^32: bound on a tile's sum of P
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr int kErrTimeout = 1;
// With segment ids, each CTA lists its visited key tiles in shared memory when
// there are at most this many key tiles (S_kv <= 262144); beyond, roles walk
// the summaries in global memory.
constexpr int kMaxListedTiles = 2048;
// Threads that read a unit's tile list (loader warp, MMA warp, softmax
// warpgroups); each arrives once when it is done with the list.
constexpr int kListReaders = 320;
// A list entry: the key tile's index | kListRaster when its keys lie in raster
// order (windows; see win_tile_bbox_kernel) | bit 30 + i when Q tile i needs
// the mask on it.
constexpr int kListTileMask = 0x1FFFFFFF;
constexpr int kListRaster = 1 << 29;

struct FwdParams {
  const int32_t* seg_q;     // [B,S_q] or null
  const int32_t* seg_kv;    // [B,S_kv] or null
  // ids: [B,n_q_tiles] {min,max,uniform,0}; window: the tiles' coordinate
  // boxes (win_tile_bbox_kernel); null with neither
  const int4* q_sum;
  const int4* kv_sum;       // [B,n_kv_tiles]
  // 3D neighbourhood window (vidattn_fwd_window), or coord_q == null: per-token
  // coordinates t << 22 | h << 11 | w, window size and volume extent per axis
  const int32_t* coord_q;   // [B,S_q]
  const int32_t* coord_kv;  // [B,S_kv]
  int win_size[3], win_extent[3], win_clamped;
  FastDiv div_wg, div_hg;   // by win_extent[2] (Wg) and win_extent[1] (Hg)
  uint16_t* out;            // bf16 [B,H,S_q,D]
  float* lse;               // fp32 [B,H,S_q]
  int* err;                 // device error word (bit kErrTimeout: a wait timed out)
  int H, S_q, S_kv;
  int n_q_tiles, n_kv_tiles;
  int n_pairs;              // 256-row query blocks per (b, h): ceil(S_q / 256)
  int n_split;              // key splits per query block (1: no split)
  int n_units;              // B * H * n_pairs * n_split work units
  // n_split > 1: per split, O / l and the log-sum-exp of each row, fp32
  // [B*H][n_split][S_q][D] and [B*H][n_split][S_q], merged by split_combine_kernel
  float* part_o;
  float* part_lse;
  int causal;               // nonzero: key j visible to query i only if j <= i + causal_off
  int causal_off;           // S_kv - S_q (the last query aligned with the last key)
  float c;                  // scale * log2(e)
  unsigned long long* trace; // VIDATTN_TRACE builds only: per-event clock64 stamps
};

// Timeline instrumentation, compiled in only with -DVIDATTN_TRACE: role r
// (0 MMA, 1/2 softmax of Q tile 0/1, 3 loader), key tile t < 64, event e < 16
// of one CTA (the middle of the grid) get a clock64() stamp.
#ifdef VIDATTN_TRACE
#define VIDATTN_TR(r, t, e)                                                        \
  do {                                                                             \
    if (trace_cta && (t) < 64) p.trace[((r) * 64 + (t)) * 16 + (e)] = clock64();   \
  } while (0)
#else
#define VIDATTN_TR(r, t, e) \
  do {                      \
  } while (0)
#endif

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kSub = D / 64;                 // 128-byte column blocks per row
  static constexpr int kSubBytes = 128 * 128;         // [128 rows][64 bf16]
  static constexpr int kTileBytes = kSub * kSubBytes; // one Q, K or V tile
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  // q_full[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] drain[1] s_free[2]
  // q_empty[1] list_full[2] list_empty[2]
  static constexpr int kNumBars = 2 + 2 * kStages + 14;
  // tmem addr, abort flag, the two lists' lengths
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kOffList = kOffMisc + 16;            // two lists of key tiles
  // per softmax warp: the ids or window coordinates of the 128 keys of the
  // masked key tile it is working on (read as int4: 16-byte aligned)
  static constexpr int kOffKinfo = (kOffList + 2 * 4 * kMaxListedTiles + 127) & ~127;
  static_assert(kOffKinfo % 16 == 0, "int4 reads of the key-info slots");
  static constexpr int kSmemBytes = kOffKinfo + 8 * kBN * 4 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "one CTA's shared memory on sm_100");
  // P in its own tensor-memory columns (D = 64, where they fit) instead of
  // over the first half of S: the next Q K^T of a tile need not wait for
  // the P V that reads its P.
  static constexpr bool kSepP = (D == 64);
  // TMEM columns: S_i at kTmemS + 128 i; P_i at kTmemP + 64 i (over S_i when
  // !kSepP); O_i at kTmemO + D i.
  static constexpr uint32_t kTmemS = 0;
  static constexpr uint32_t kTmemP = kSepP ? 256 : 0;
  static constexpr uint32_t kPStride = kSepP ? 64 : 128;
  static constexpr uint32_t kTmemO = kSepP ? 384 : 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBN, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
};

// Bounded wait on an mbarrier phase.  Returns false if the CTA has aborted or
// the wait exceeded kWaitTimeoutNs (then it sets the abort flag and the
// device error word).  Every thread that calls it observes the phase itself.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity,
                                           volatile int* abort_flag, int* err,
                                           uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      // give up at once if this CTA, or any CTA of this launch, already did
      if (*abort_flag || *reinterpret_cast<volatile int*>(err)) {
        *abort_flag = 1;
        return false;
      }
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > timeout_ns) {
        *abort_flag = 1;
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
}

// The same, with one outcome for the whole warp (needed before the
// warp-collective tcgen05.ld/st).
__device__ __forceinline__ bool warp_wait_phase(uint32_t bar, uint32_t parity,
                                                volatile int* abort_flag, int* err,
                                                uint64_t timeout_ns = kWaitTimeoutNs) {
  const bool ok = wait_phase(bar, parity, abort_flag, err, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// Key tiles visited by a CTA whose query ids span [qmin, qmax]: every tile
// without ids; with ids, the tiles whose id range intersects [qmin, qmax].
// Every role of the CTA walks the same sequence.
struct KvWalk {
  const int4* kv_sum;   // this batch's summaries, or null
  int n_kv;
  int qmin, qmax;
  __device__ __forceinline__ int next(int j) const {
    if (kv_sum == nullptr) return j;
    for (; j < n_kv; ++j) {
      const int4 s = __ldg(kv_sum + j);
      if (!(s.y < qmin || s.x > qmax)) return j;
    }
    return n_kv;
  }
};

// ------------------------------------------------- 3D neighbourhood window
// On each axis the window of a query at coordinate c spans
// [start, start + size - 1], start = c - (size - 1) / 2, pushed into
// [0, extent - size] when clamped (every query then sees size keys per axis).
__device__ __forceinline__ int win_start(int c, int size, int extent, int clamped) {
  int s = c - (size - 1) / 2;
  if (clamped) s = max(min(s, extent - size), 0);
  return s;
}
__device__ __forceinline__ int coord_axis(uint32_t c, int a) {
  return a == 0 ? int(c >> 22) : (a == 1 ? int((c >> 11) & 2047u) : int(c & 2047u));
}
// Window starts of one query row.
struct WinRow {
  int s[3];
};
__device__ __forceinline__ WinRow win_row(const FwdParams& p, uint32_t qc) {
  WinRow r;
#pragma unroll
  for (int a = 0; a < 3; ++a)
    r.s[a] = win_start(coord_axis(qc, a), p.win_size[a], p.win_extent[a], p.win_clamped);
  return r;
}
__device__ __forceinline__ bool win_has(const FwdParams& p, const WinRow& r, uint32_t kc) {
  bool in = true;
#pragma unroll
  for (int a = 0; a < 3; ++a)
    in = in && uint32_t(coord_axis(kc, a) - r.s[a]) < uint32_t(p.win_size[a]);
  return in;
}
// Tile boxes: field a of the int4 packs lo | hi << 16 for axis a.
__device__ __forceinline__ int box_lo(int4 b, int a) {
  return (a == 0 ? b.x : (a == 1 ? b.y : b.z)) & 0xFFFF;
}
__device__ __forceinline__ int box_hi(int4 b, int a) {
  return (a == 0 ? b.x : (a == 1 ? b.y : b.z)) >> 16;
}
// Could some query of the two Q tiles (boxes qa, qb) see some key of a K tile
// with box kb?  (Its box meets the union of their windows on every axis.)
__device__ __forceinline__ bool win_tile_meets(const FwdParams& p, int4 qa, int4 qb, int4 kb) {
  bool meets = true;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int qlo = min(box_lo(qa, a), box_lo(qb, a)), qhi = max(box_hi(qa, a), box_hi(qb, a));
    const int u_lo = win_start(qlo, p.win_size[a], p.win_extent[a], p.win_clamped);
    const int u_hi = win_start(qhi, p.win_size[a], p.win_extent[a], p.win_clamped) +
                     p.win_size[a] - 1;
    meets = meets && box_hi(kb, a) >= u_lo && box_lo(kb, a) <= u_hi;
  }
  return meets;
}
// Does every query of a Q tile (box qa) see every key of a K tile (box kb)?
// (The K box lies inside the intersection of the queries' windows.)
__device__ __forceinline__ bool win_tile_full(const FwdParams& p, int4 qa, int4 kb) {
  bool full = true;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int i_lo = win_start(box_hi(qa, a), p.win_size[a], p.win_extent[a], p.win_clamped);
    const int i_hi = win_start(box_lo(qa, a), p.win_size[a], p.win_extent[a], p.win_clamped) +
                     p.win_size[a] - 1;
    full = full && box_lo(kb, a) >= i_lo && box_hi(kb, a) <= i_hi;
  }
  return full;
}

// Sets bits [lo, hi) of a 128-bit mask.
__device__ __forceinline__ void set_bit_range(uint32_t (&mb)[4], int lo, int hi) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = max(lo - 32 * k, 0), e = min(hi - 32 * k, 32);
    if (a < e) mb[k] |= (e == 32 ? 0xFFFFFFFFu : ((1u << e) - 1u)) & ~((1u << a) - 1u);
  }
}

constexpr int kMaxRuns = 16;   // runs per key tile handled run by run

// The mask of one query row over a masked key tile, bit x of word x/32 set
// when key x of the tile is visible: x < n_lim (the key exists and lies
// within the causal limit) and the key has the row's id (mode 1) or lies in
// its window (mode 2: window starts ws0..2, sizes k0..2).  kinfo: the 128
// keys' ids or coordinates, staged in this warp's shared memory by the
// caller (unused in mode 0).  Called by the whole warp.
//
// The keys of a tile fall into runs: consecutive keys with one id, or with
// one (t, h) and consecutive w (a row of the volume in raster order).  A
// row's visible keys in a run are one contiguous range, so with few runs the
// mask is built run by run; otherwise key by key.
__device__ __forceinline__ uint4 tile_mask(const int32_t* kinfo, int mode, int my_seg, int ws0,
                                        int ws1, int ws2, int k0, int k1, int k2, int n_lim) {
  const int lane = threadIdx.x & 31;
  uint32_t mb[4] = {0u, 0u, 0u, 0u};
  if (mode == 0) {
    set_bit_range(mb, 0, n_lim);
    return make_uint4(mb[0], mb[1], mb[2], mb[3]);
  }
  const bool ids = mode == 1;
  // run starts (the same for every row of the warp)
  uint32_t starts[4];
  int n_runs = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int x = lane + 32 * m;
    const int32_t cur = kinfo[x];
    const int32_t prev = kinfo[x > 0 ? x - 1 : 0];
    const bool cont = ids ? (prev == cur)
                          : (uint32_t(cur) == uint32_t(prev) + 1u && (cur & 2047) != 0);
    starts[m] = __ballot_sync(0xFFFFFFFFu, x == 0 || !cont);
    n_runs += __popc(starts[m]);
  }
  if (n_runs <= kMaxRuns) {
    // walk the runs in order: [xa, xb)
    uint32_t rest[4] = {starts[0] & ~1u, starts[1], starts[2], starts[3]};
    int xa = 0;
    for (int r = 0; r < n_runs; ++r) {
      int xb = kBN;
#pragma unroll
      for (int k = 3; k >= 0; --k)
        if (rest[k]) xb = 32 * k + __ffs(rest[k]) - 1;
      const int32_t c0 = kinfo[xa];
      if (ids) {
        if (c0 == my_seg) set_bit_range(mb, xa, xb);
      } else {
        const uint32_t u = uint32_t(c0);
        if (uint32_t(int(u >> 22) - ws0) < uint32_t(k0) &&
            uint32_t(int((u >> 11) & 2047u) - ws1) < uint32_t(k1)) {
          const int w0 = int(u & 2047u);
          const int lo = xa + max(ws2 - w0, 0);
          const int hi = xa + min(ws2 + k2 - w0, xb - xa);
          if (lo < hi) set_bit_range(mb, lo, hi);
        }
      }
      // clear the next run's start bit (selects: no dynamic register index)
      const uint32_t clear = ~(1u << (xb & 31));
#pragma unroll
      for (int k = 0; k < 4; ++k) rest[k] &= ((xb >> 5) == k) ? clear : 0xFFFFFFFFu;
      xa = xb;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t bits = 0u;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        const int4 v = *reinterpret_cast<const int4*>(kinfo + 32 * k + x);
        const int vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t u = uint32_t(vv[e]);
          const bool in = ids ? (vv[e] == my_seg)
                              : (uint32_t(int(u >> 22) - ws0) < uint32_t(k0) &&
                                 uint32_t(int((u >> 11) & 2047u) - ws1) < uint32_t(k1) &&
                                 uint32_t(int(u & 2047u) - ws2) < uint32_t(k2));
          bits |= (in ? 1u : 0u) << (x + e);
        }
      }
      mb[k] = bits;
    }
  }
  uint32_t lim[4] = {0u, 0u, 0u, 0u};
  set_bit_range(lim, 0, n_lim);
  return make_uint4(mb[0] & lim[0], mb[1] & lim[1], mb[2] & lim[2], mb[3] & lim[3]);
}

// The same as a call, so that its registers do not weigh on the softmax's
// where masked tiles are rare.
__device__ __noinline__ uint4 tile_mask_call(const int32_t* kinfo, int mode, int my_seg, int ws0,
                                             int ws1, int ws2, int k0, int k1, int k2,
                                             int n_lim) {
  return tile_mask(kinfo, mode, my_seg, ws0, ws1, ws2, k0, k1, k2, n_lim);
}

// Window variant: the mask of one query row (window starts ws0..2, sizes
// k0..2) over key tile j whose keys lie in raster order in a volume of rows
// of Wg tokens and Hg rows per frame: key x of the tile is token j*128 + x at
// (t, h, w) = its raster position, so the tile's keys are the runs of the
// (t, h) rows it crosses, and a row sees the keys of a run whose (t, h) is in
// its window, w in [ws2, ws2 + k2).  Keys at or past n_lim are hidden.  The
// same bits as tile_mask's in mode 2, from the tile index alone.
__device__ __forceinline__ uint4 raster_mask(const FwdParams& p, int j, int n_lim, int ws0,
                                            int ws1, int ws2) {
  const int Hg = p.win_extent[1], Wg = p.win_extent[2];
  const int k0 = p.win_size[0], k1 = p.win_size[1], k2 = p.win_size[2];
  const int k_first = j * kBN;
  const int r0 = int(fastdiv(uint32_t(k_first), p.div_wg));   // (t, h) row of the first key
  int xa = r0 * Wg - k_first;                  // tile offset of that row's w = 0 (<= 0)
  int t = int(fastdiv(uint32_t(r0), p.div_hg));
  int h = r0 - t * Hg;
  const int wlo = max(ws2, 0), whi = min(ws2 + k2, Wg);
  // the mask as two 64-bit halves: bits [a, e) of a half, 0 <= a < e <= 64,
  // are (~0 >> (64 - (e - a))) << a
  uint64_t m01 = 0, m23 = 0;
  for (; xa < n_lim; xa += Wg) {
    if (uint32_t(t - ws0) < uint32_t(k0) && uint32_t(h - ws1) < uint32_t(k1)) {
      const int lo = max(xa + wlo, 0);
      const int hi = min(xa + whi, n_lim);
      const int a0 = min(lo, 64), e0 = min(hi, 64);
      const int a1 = max(lo, 64) - 64, e1 = max(hi, 64) - 64;
      if (a0 < e0) m01 |= (~0ull >> (64 - (e0 - a0))) << a0;
      if (a1 < e1) m23 |= (~0ull >> (64 - (e1 - a1))) << a1;
    }
    if (++h == Hg) {
      h = 0;
      ++t;
    }
  }
  return make_uint4(uint32_t(m01), uint32_t(m01 >> 32), uint32_t(m23), uint32_t(m23 >> 32));
}

// One thread's row of a 128-column S tile from tensor memory.
__device__ __forceinline__ void load_s_row(uint32_t taddr, float (&s)[kBN]) {
  uint32_t sr[4][32];
#pragma unroll
  for (int k = 0; k < 4; ++k) tmem_ld32(taddr + 32 * k, sr[k]);
  tmem_ld_wait();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    reg_fence(sr[k]);
#pragma unroll
    for (int x = 0; x < 32; ++x) s[32 * k + x] = __uint_as_float(sr[k][x]);
  }
}

// Maximum of a row: four independent three-input max chains, 16 deep.
__device__ __forceinline__ float row_max(const float (&s)[kBN]) {
  float a[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
  for (int x = 8; x < kBN; x += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = max3f(a[k], s[x + 2 * k], s[x + 2 * k + 1]);
  }
  return max3f(a[0], a[1], fmaxf(a[2], a[3]));
}

// p = 2^(c*s - m) for a row of 128 scores: per 16 keys, the first 16 - kEmu
// on the MUFU unit (ex2), the last kEmu on the FMA pipe (exp2_poly2).  The
// bf16-rounded p go to pk (two per word, the layout of P in tensor memory);
// returns the fp32 sum of p (four packed partial sums).  kMasked: keys whose
// bit in mb is clear get p = 0 (whatever their score).
template <int kEmu, bool kMasked = false>
__device__ __forceinline__ float exp_tile(const float (&s)[kBN], float c, float m,
                                          uint32_t (&pk)[2][32], const uint32_t* mb = nullptr) {
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int x = 0; x < kBN; x += 2) {
    const float2 arg = ffma2(make_float2(s[x], s[x + 1]), c2, nm2);
    float2 e;
    if ((x & 15) < 16 - kEmu) {
      e.x = ex2(arg.x);
      e.y = ex2(arg.y);
    } else {
      e = exp2_poly2(arg);
    }
    if constexpr (kMasked) {
      e.x = ((mb[x >> 5] >> (x & 31)) & 1u) ? e.x : 0.f;
      e.y = ((mb[x >> 5] >> ((x + 1) & 31)) & 1u) ? e.y : 0.f;
    }
    acc[(x >> 1) & 3] = fadd2(acc[(x >> 1) & 3], e);
    pk[x >> 6][(x >> 1) & 31] = pack_bf16x2(e.x, e.y);
  }
  const float2 s01 = fadd2(acc[0], acc[1]), s23 = fadd2(acc[2], acc[3]);
  const float2 s03 = fadd2(s01, s23);
  return s03.x + s03.y;
}

// p = 2^(c*s - m) for keys [kX0, kX0 + 32) of the row (one 32-bit mask
// word): the bf16 pairs into pk[kX0/2 .. kX0/2 + 16); returns their fp32 sum.
// Keys whose bit in mk is clear get p = 0.
template <int kEmu, int kX0>
__device__ __forceinline__ float exp_chunk_masked(const float (&s)[kBN], float c, float m,
                                                  uint32_t mk, uint32_t (&pk)[2][32]) {
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int x = kX0; x < kX0 + 32; x += 2) {
    const float s0 = ((mk >> (x & 31)) & 1u) ? s[x] : -INFINITY;
    const float s1 = ((mk >> ((x + 1) & 31)) & 1u) ? s[x + 1] : -INFINITY;
    const float2 arg = ffma2(make_float2(s0, s1), c2, nm2);
    float2 e;
    if ((x & 15) < 16 - kEmu) {
      e.x = ex2(arg.x);
      e.y = ex2(arg.y);
    } else {
      e = exp2_poly2(arg);
    }
    acc[(x >> 1) & 1] = fadd2(acc[(x >> 1) & 1], e);
    pk[x >> 6][(x >> 1) & 31] = pack_bf16x2(e.x, e.y);
  }
  const float2 s01 = fadd2(acc[0], acc[1]);
  return s01.x + s01.y;
}

// Causal limit: one past the last key tile any query row of CTA `pair` can
// see (all tiles when not causal; 0 when no row sees any key).
__device__ __forceinline__ int causal_end(const FwdParams& p, int pair) {
  if (!p.causal) return p.n_kv_tiles;
  const int max_row = min(pair * 2 * kBM + 2 * kBM - 1, p.S_q - 1);
  const int last_key = max_row + p.causal_off;
  if (last_key < 0) return 0;
  return min(p.n_kv_tiles, last_key / kBN + 1);
}

// Causal limit: does Q tile qi of CTA `pair` see only part of key tile j
// (some key of the tile lies after its first row's limit)?  Then that tile
// takes the masked path for that Q tile.
__device__ __forceinline__ bool causal_partial(const FwdParams& p, int pair, int qi, int j) {
  if (!p.causal) return false;
  const int r0 = pair * 2 * kBM + qi * kBM;
  return j * kBN + kBN - 1 > r0 + p.causal_off;
}

// The key-tile walk of CTA (b, pair) and, optionally, the id summary of one
// of its two query tiles (qi), read from the classifier's output.  Each role
// builds its own copy, so nothing stays live across the role branches.
__device__ __forceinline__ KvWalk make_walk(const FwdParams& p, int b, int pair, int qi = -1,
                                            int4* q_summary = nullptr) {
  KvWalk walk{nullptr, causal_end(p, pair), 0, 0};
  if (p.q_sum == nullptr) {
    if (q_summary) *q_summary = make_int4(0, 0, 1, 0);
    return walk;
  }
  const int qt0 = 2 * pair;
  const int4* qsum_b = p.q_sum + static_cast<int64_t>(b) * p.n_q_tiles;
  const int4 q0 = __ldg(qsum_b + qt0);
  const int4 q1 = (qt0 + 1 < p.n_q_tiles) ? __ldg(qsum_b + qt0 + 1) : q0;
  if (q_summary) *q_summary = (qi == 1) ? q1 : q0;
  if (p.coord_q == nullptr) {   // ids: walk the tiles whose id range meets the queries'
    walk.kv_sum = p.kv_sum + static_cast<int64_t>(b) * p.n_kv_tiles;
    walk.qmin = min(q0.x, q1.x);
    walk.qmax = max(q0.y, q1.y);
  }
  return walk;
}

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t sQ, uint32_t sK) {
  using C = FwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * C::kSubBytes + (kk % 4) * 32;
    const uint64_t a = smem_desc_sw128(sQ + off, 16, 1024);
    const uint64_t b = smem_desc_sw128(sK + off, 16, 1024);
    mma_ss_elect(d_tmem, a, b, C::kIdescQK, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t sV,
                                         bool accumulate) {
  using C = FwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    // V is [keys][D] with D contiguous: MN-major for the B operand (N = D).
    // 16 keys = two 8-row swizzle atoms (SBO = 1024); D/64 column blocks
    // are kSubBytes apart (LBO).
    const uint64_t b = smem_desc_sw128(sV + kk * 2048, C::kSubBytes, 1024);
    mma_ts_elect(d_tmem, p_tmem + kk * 8, b, C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One work unit of the persistent kernel: (b, h, 256-row query block `pair`,
// key split `split` of n_split).
struct Unit {
  int b, h, pair, split;
};
// Units are numbered split fastest, then query block, then head: one head's
// units run close together in time (its K and V stay in L2).  With the
// causal limit the query blocks of a head go longest first (the last block
// sees the most keys), so no long unit trails at the end of the launch.
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  Unit x;
  x.split = u % p.n_split;
  const int r = u / p.n_split;
  const int pp = r % p.n_pairs;
  const int bh = r / p.n_pairs;
  x.b = bh / p.H;
  x.h = bh - x.b * p.H;
  x.pair = p.causal ? p.n_pairs - 1 - pp : pp;
  return x;
}

// The key tiles a unit visits: positions [t0, t1) of the pair's visit
// sequence (its listed tiles, or every tile below the causal end, or the
// global walk with ids beyond the list's capacity, where n_split is 1).
struct UnitSched {
  const int* list;   // the unit's listed tiles, or null
  int t0, t1;
  int n_kv;          // one past the last key tile any row of the pair can see
  KvWalk walk;
  // j of position t (prev_j: j of position t - 1, or t0 - 1 at the start);
  // n_kv once the unit's range is done
  __device__ __forceinline__ int tile(int t, int prev_j) const {
    if (t >= t1) return n_kv;
    if (list != nullptr) return list[t] & kListTileMask;
    return walk.next(prev_j + 1);
  }
};

__device__ __forceinline__ UnitSched unit_sched(const FwdParams& p, const Unit& x,
                                                const int* list, int n_list) {
  UnitSched s;
  s.list = list;
  s.walk = make_walk(p, x.b, x.pair);
  s.n_kv = s.walk.n_kv;
  // positions of the whole pair: listed tiles, the global walk (ids beyond
  // the list's capacity: its length is not known up front; n_split is 1) or
  // every tile below the causal end
  const int total = list != nullptr ? n_list : (s.walk.kv_sum != nullptr ? INT_MAX : s.n_kv);
  if (p.n_split == 1) {
    s.t0 = 0;
    s.t1 = total;
  } else {
    s.t0 = int((int64_t(total) * x.split) / p.n_split);
    s.t1 = int((int64_t(total) * (x.split + 1)) / p.n_split);
  }
  return s;
}

// kEmu: exponentials per 16 keys computed on the FMA pipe instead of MUFU.
// kMaskFast: masked key tiles (D = 128) take the running-offset path with
// their hidden keys' scores set to -inf, instead of the two-pass exact path
// (the variant for 3D neighbourhood windows, where nearly every visited tile
// is masked; elsewhere the extra code costs the unmasked tiles registers).
//
// kSplit: the launch splits the keys (FwdParams::n_split > 1); the epilogue
// writes each split's partial result for split_combine_kernel instead of out
// and lse.
// kPersist: the grid holds at most one CTA per SM, and CTA i works on units
// i, i + gridDim.x, ...  Every barrier phase runs on across units, so the
// loader fetches the next unit's Q and first K/V tiles and the MMA warp
// issues its first Q K^T while the softmax warps still write the previous
// unit's output.  Otherwise one CTA per unit, scheduled by the hardware as
// SMs free up.
template <int D, int kEmu, bool kMaskFast, bool kPersist, bool kSplit>
__global__ void __launch_bounds__(kFwdThreads, 1)
    vidattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t sbase = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_base);

  // A wait of an earlier CTA timed out: the results are already invalid,
  // so later CTAs end at once instead of timing out one by one.
  if (*reinterpret_cast<volatile int*>(p.err) != 0) return;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the units of this CTA: every gridDim.x-th from blockIdx.x when
  // persistent; else the grid holds one CTA per unit and the loops below run
  // once (a trip count the compiler sees, so nothing carries across units)
  const int u_end = kPersist ? p.n_units : int(blockIdx.x) + 1;
  const int u_step = kPersist ? int(gridDim.x) : 1;

  const uint32_t sQ[2] = {sbase + C::kOffQ, sbase + C::kOffQ + C::kTileBytes};
  auto sKV = [&](int s) { return sbase + C::kOffKV + s * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kOffBar + 8 * i; };
  auto q_full = [&](int i) { return bar(i); };
  auto kv_full = [&](int s) { return bar(2 + s); };
  auto kv_empty = [&](int s) { return bar(2 + C::kStages + s); };
  auto s_full = [&](int i) { return bar(2 + 2 * C::kStages + i); };
  auto p_full = [&](int i) { return bar(4 + 2 * C::kStages + i); };
  auto o_full = [&](int i) { return bar(6 + 2 * C::kStages + i); };
  const uint32_t drain_bar = bar(8 + 2 * C::kStages);
  auto s_free = [&](int i) { return bar(9 + 2 * C::kStages + i); };
  // the Q tiles may be overwritten (every Q K^T of the unit has run)
  const uint32_t q_empty = bar(11 + 2 * C::kStages);
  // tile lists, double-buffered: written (list_full) / read by every role (list_empty)
  auto list_full = [&](int i) { return bar(12 + 2 * C::kStages + i); };
  auto list_empty = [&](int i) { return bar(14 + 2 * C::kStages + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* list_count = reinterpret_cast<int*>(smem + C::kOffMisc + 8);   // [2]
  int* list_base = reinterpret_cast<int*>(smem + C::kOffList);          // [2][kMaxListedTiles]

  if (threadIdx.x == 0) {
    mbar_init(q_full(0), 1);
    mbar_init(q_full(1), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), 128);
      mbar_init(o_full(i), 1);
      mbar_init(s_free(i), 128);
      mbar_init(list_full(i), 32);
      mbar_init(list_empty(i), kListReaders);
    }
    mbar_init(drain_bar, 1);
    mbar_init(q_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  const bool has_sum = p.q_sum != nullptr;      // tile summaries: ids or window boxes
  const bool has_win = p.coord_q != nullptr;
  const bool has_seg = has_sum && !has_win;
  // With summaries, warp 10 lists each unit's visited key tiles (id ranges or
  // window boxes that meet its queries') with per-Q-tile mask bits, so no
  // role touches global memory to find its next tile; beyond the list's
  // capacity the roles walk the summaries in global memory.
  const bool listed = has_sum && p.n_kv_tiles <= kMaxListedTiles;
#ifdef VIDATTN_TRACE
  const bool trace_cta = p.trace != nullptr && blockIdx.x == gridDim.x / 2;
#endif
  // list of the k-th unit of this CTA, once warp 10 has written it
  auto wait_list = [&](int k, const int** list, int* n_list) -> bool {
    *list = nullptr;
    *n_list = 0;
    if (!listed) return true;
    const int buf = k & 1;
    if (!warp_wait_phase(list_full(buf), uint32_t(k >> 1) & 1u, abort_flag, p.err)) return false;
    *list = list_base + buf * kMaxListedTiles;
    *n_list = *reinterpret_cast<volatile int*>(list_count + buf);
    return true;
  };
  auto release_list = [&](int k) {
    if (listed) mbar_arrive(list_empty(k & 1));
  };

  // Register split: the launch gives 168 per thread (384 x 168 = 64512);
  // warpgroup 2 (MMA, TMA, list builder, idle warp) drops so the two softmax
  // warpgroups can rise.  Per variant, a split without register spills
  // (ptxas, for the default kEmu of each head dim): D = 128: 128 x 128 +
  // 256 x 184 = 63488; D = 64 persistent: 128 x 96 + 256 x 200 = 63488; the
  // others (D = 64, the window variant, whose softmax also holds the mask):
  // 128 x 104 + 256 x 192 = 62464; all <= 64512.  Each warpgroup executes
  // its setmaxnreg at the head of its own branch.
  if (warp >= 8) {
  if constexpr (D == 128 && !kMaskFast) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 128;" ::: "memory");
  } else if constexpr (kPersist) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;" ::: "memory");
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 104;" ::: "memory");
  }
  if (warp == 9) {
    // ------------------------------------------------------------ TMA loads
    // the whole warp runs the loop; one elected lane issues
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    int n = 0;    // K/V loads issued (ring position), over all units
    int kq = 0;   // units with at least one tile so far (Q loads)
    bool ok = true;
    for (int u = blockIdx.x, k = 0; ok && u < u_end; u += u_step, ++k) {
      const int* list;
      int n_list;
      ok = wait_list(k, &list, &n_list);
      if (!ok) break;
      const Unit x = decode_unit(p, u);
      const UnitSched sched = unit_sched(p, x, list, n_list);
      const int bh = x.b * p.H + x.h;
      const int m0 = x.pair * 2 * kBM;
      int t = sched.t0;
      int j = sched.tile(t, t - 1);
      if (j < sched.n_kv) {
        if (kq > 0) ok = warp_wait_phase(q_empty, uint32_t(kq - 1) & 1u, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(q_full(0), C::kTileBytes);
        for (int s = 0; s < C::kSub; ++s)
          tma_load_3d_elect(sQ[0] + s * C::kSubBytes, &tm_q, q_full(0), s * 64, m0, bh);
        bool first = true;
        while (ok && j < sched.n_kv) {
          for (int which = 0; which < 2 && ok; ++which) {   // K_j then V_j
            const int st = n % C::kStages;
            VIDATTN_TR(3, n, 0);
            ok = warp_wait_phase(kv_empty(st), ((n / C::kStages) & 1) ^ 1, abort_flag, p.err);
            VIDATTN_TR(3, n, 1);
            if (!ok) break;
            mbar_arrive_expect_tx_elect(kv_full(st), C::kTileBytes);
            for (int s = 0; s < C::kSub; ++s)
              tma_load_3d_elect(sKV(st) + s * C::kSubBytes, which ? &tm_v : &tm_k, kv_full(st),
                                s * 64, j * kBN, bh);
            ++n;
            if (first) {
              first = false;
              mbar_arrive_expect_tx_elect(q_full(1), C::kTileBytes);
              for (int s = 0; s < C::kSub; ++s)
                tma_load_3d_elect(sQ[1] + s * C::kSubBytes, &tm_q, q_full(1), s * 64, m0 + kBM,
                                  bh);
            }
          }
          j = sched.tile(++t, j);
        }
        ++kq;
      }
      __syncwarp();
      release_list(k);
    }
    if (!ok) {
      // Let the loads already in flight land before the CTA can exit.
      for (int k = (n > C::kStages ? n - C::kStages : 0); k < n; ++k) {
        const int st = k % C::kStages;
        volatile int never = 0;
        warp_wait_phase(kv_full(st), (k / C::kStages) & 1, &never, p.err);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ------------------------------------------------------- tensor core
    // the whole warp runs the loop; one elected lane issues
    auto stage = [&](int idx) { return idx % C::kStages; };
    auto par = [&](int idx) { return uint32_t(idx / C::kStages) & 1u; };
    int n = 0;    // K/V tiles consumed (ring position), over all units
    int T = 0;    // key tiles done by this CTA, over all units (barrier parities)
    int kq = 0;   // units with at least one tile so far
    bool ok = true;
    for (int u = blockIdx.x, k = 0; ok && u < u_end; u += u_step, ++k) {
      const int* list;
      int n_list;
      ok = wait_list(k, &list, &n_list);
      if (!ok) break;
      const Unit x = decode_unit(p, u);
      const UnitSched sched = unit_sched(p, x, list, n_list);
      int t = sched.t0;
      int j = sched.tile(t, t - 1);
      if (j < sched.n_kv) {
        const uint32_t qpar = uint32_t(kq) & 1u;
        if (C::kSepP) {
          // Order per tile t: S0 = Q0 K_{t+1}^T once S0_t is read, O0 += P0 V_t,
          // S1 = Q1 K_{t+1}^T once S1_t is read, O1 += P1 V_t.  K_t is load 2t
          // and V_t load 2t+1 of the ring.
          ok = warp_wait_phase(q_full(0), qpar, abort_flag, p.err);
          ok = ok && warp_wait_phase(kv_full(stage(n)), par(n), abort_flag, p.err);
          // S0 of the previous unit's last tile has been read
          ok = ok && (T == 0 || warp_wait_phase(s_free(0), uint32_t(T - 1) & 1u, abort_flag, p.err));
          const int k0 = n++;
          if (ok) {
            tc_fence_after();
            issue_qk<D>(tmem + C::kTmemS, sQ[0], sKV(stage(k0)));
            mma_commit_elect(s_full(0));
            ok = warp_wait_phase(q_full(1), qpar, abort_flag, p.err);
            ok = ok && (T == 0 || warp_wait_phase(s_free(1), uint32_t(T - 1) & 1u, abort_flag, p.err));
          }
          if (ok) {
            tc_fence_after();
            issue_qk<D>(tmem + C::kTmemS + 128, sQ[1], sKV(stage(k0)));
            mma_commit_elect(s_full(1));
            mma_commit_elect(kv_empty(stage(k0)));
          }
          bool first = true;
          while (ok) {
            const int jn = sched.tile(t + 1, j);
            const bool more = jn < sched.n_kv;
            if (!more) mma_commit_elect(q_empty);   // the unit's last Q K^T is issued
            const int vi = n++;
            VIDATTN_TR(0, T, 0);
            // both tiles' data first (see the aliased loop)
            ok = warp_wait_phase(kv_full(stage(vi)), par(vi), abort_flag, p.err);
            int kn = 0;
            if (ok && more) {
              kn = n++;
              ok = warp_wait_phase(kv_full(stage(kn)), par(kn), abort_flag, p.err);
            }
            if (!ok) break;
            if (more) {
              ok = warp_wait_phase(s_free(0), uint32_t(T) & 1u, abort_flag, p.err);
              VIDATTN_TR(0, T, 1);
              if (!ok) break;
              tc_fence_after();
              issue_qk<D>(tmem + C::kTmemS, sQ[0], sKV(stage(kn)));
              mma_commit_elect(s_full(0));
              VIDATTN_TR(0, T, 2);
            }
            ok = warp_wait_phase(p_full(0), uint32_t(T) & 1u, abort_flag, p.err);
            VIDATTN_TR(0, T, 3);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D>(tmem + C::kTmemO, tmem + C::kTmemP, sKV(stage(vi)), !first);
            mma_commit_elect(o_full(0));
            VIDATTN_TR(0, T, 4);
            if (more) {
              ok = warp_wait_phase(s_free(1), uint32_t(T) & 1u, abort_flag, p.err);
              VIDATTN_TR(0, T, 5);
              if (!ok) break;
              tc_fence_after();
              issue_qk<D>(tmem + C::kTmemS + 128, sQ[1], sKV(stage(kn)));
              mma_commit_elect(s_full(1));
              mma_commit_elect(kv_empty(stage(kn)));
              VIDATTN_TR(0, T, 6);
            }
            ok = warp_wait_phase(p_full(1), uint32_t(T) & 1u, abort_flag, p.err);
            VIDATTN_TR(0, T, 7);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D>(tmem + C::kTmemO + D, tmem + C::kTmemP + C::kPStride, sKV(stage(vi)),
                        !first);
            mma_commit_elect(o_full(1));
            mma_commit_elect(kv_empty(stage(vi)));
            VIDATTN_TR(0, T, 8);
            ++T;
            first = false;
            if (!more) break;
            j = jn;
            ++t;
          }
        } else {
          ok = warp_wait_phase(q_full(0), qpar, abort_flag, p.err);
          const int ks = stage(n);
          ok = ok && warp_wait_phase(kv_full(ks), par(n), abort_flag, p.err);
          ++n;
          if (ok) {
            tc_fence_after();
            issue_qk<D>(tmem + C::kTmemS, sQ[0], sKV(ks));
            mma_commit_elect(s_full(0));
            ok = warp_wait_phase(q_full(1), qpar, abort_flag, p.err);
          }
          if (ok) {
            tc_fence_after();
            issue_qk<D>(tmem + (C::kTmemS + 128), sQ[1], sKV(ks));
            mma_commit_elect(s_full(1));
            mma_commit_elect(kv_empty(ks));
          }
          bool first = true;
          while (ok) {
            const int jn = sched.tile(t + 1, j);
            const bool more = jn < sched.n_kv;
            if (!more) mma_commit_elect(q_empty);   // the unit's last Q K^T is issued
            const int vs = stage(n);
            VIDATTN_TR(0, T, 0);
            ok = warp_wait_phase(kv_full(vs), par(n), abort_flag, p.err);
            ++n;
            if (!ok) break;
            // Check that K_{t+1} has landed now, while this warp waits anyway,
            // instead of between dependent MMAs (an mbarrier read is slow while
            // a shared-memory-bound Q K^T runs).
            int ks2 = 0;
            if (more) {
              ks2 = stage(n);
              ok = warp_wait_phase(kv_full(ks2), par(n), abort_flag, p.err);
              ++n;
              if (!ok) break;
            }
            ok = warp_wait_phase(p_full(0), uint32_t(T) & 1u, abort_flag, p.err);
            VIDATTN_TR(0, T, 3);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D>(tmem + C::kTmemO, tmem + C::kTmemS, sKV(vs), !first);
            mma_commit_elect(o_full(0));
            VIDATTN_TR(0, T, 4);
            if (more) {
              tc_fence_after();
              issue_qk<D>(tmem + C::kTmemS, sQ[0], sKV(ks2));
              mma_commit_elect(s_full(0));
              VIDATTN_TR(0, T, 2);
            }
            ok = warp_wait_phase(p_full(1), uint32_t(T) & 1u, abort_flag, p.err);
            VIDATTN_TR(0, T, 7);
            if (!ok) break;
            tc_fence_after();
            issue_pv<D>(tmem + (C::kTmemO + D), tmem + (C::kTmemS + 128), sKV(vs), !first);
            mma_commit_elect(o_full(1));
            mma_commit_elect(kv_empty(vs));
            ++T;
            first = false;
            if (!more) break;
            issue_qk<D>(tmem + (C::kTmemS + 128), sQ[1], sKV(ks2));
            mma_commit_elect(s_full(1));
            mma_commit_elect(kv_empty(ks2));
            VIDATTN_TR(0, T, 8);
            j = jn;
            ++t;
          }
        }
        ++kq;
      }
      __syncwarp();
      release_list(k);
    }
    // Every MMA issued above has finished before TMEM is released.
    mma_commit_elect(drain_bar);
    volatile int never = 0;
    warp_wait_phase(drain_bar, 0, &never, p.err);
    __syncwarp();
  } else if (warp == 10 && listed) {
    // ------------------------------------------------------- tile lists
    // For each unit of this CTA: the key tiles the pair visits (id ranges or
    // window boxes that meet its queries'; with the causal limit, below its
    // end), entry = j | bit 30 + i when Q tile i needs the mask on tile j.
    bool ok = true;
    const bool ragged = (p.S_kv % kBN) != 0;
    for (int u = blockIdx.x, k = 0; u < u_end; u += u_step, ++k) {
      const int buf = k & 1;
      if (k >= 2) ok = warp_wait_phase(list_empty(buf), uint32_t((k >> 1) - 1) & 1u, abort_flag, p.err);
      if (!ok) break;
      const Unit x = decode_unit(p, u);
      int4 q0, q1;
      const KvWalk w = make_walk(p, x.b, x.pair, 0, &q0);
      make_walk(p, x.b, x.pair, 1, &q1);
      const int n_kv = w.n_kv;
      const int4* kv_sum_b = p.kv_sum + static_cast<int64_t>(x.b) * p.n_kv_tiles;
      int* list = list_base + buf * kMaxListedTiles;
      int cnt = 0;
      for (int c0 = 0; c0 < n_kv; c0 += 32) {
        const int jj = c0 + lane;
        bool act = false;
        int entry = 0;
        if (jj < n_kv) {
          const int4 ks = __ldg(kv_sum_b + jj);
          const bool last_ragged = ragged && jj == p.n_kv_tiles - 1;
          bool m0, m1;
          if (has_win) {
            act = win_tile_meets(p, q0, q1, ks);
            m0 = last_ragged || !win_tile_full(p, q0, ks);
            m1 = last_ragged || !win_tile_full(p, q1, ks);
          } else {
            act = !(ks.y < w.qmin || ks.x > w.qmax);
            m0 = last_ragged || !(q0.z && ks.z && q0.x == ks.x) || causal_partial(p, x.pair, 0, jj);
            m1 = last_ragged || !(q1.z && ks.z && q1.x == ks.x) || causal_partial(p, x.pair, 1, jj);
          }
          entry = jj | (m0 ? (1 << 30) : 0) | (m1 ? int(1u << 31) : 0) |
                  ((has_win && ks.w == 1) ? kListRaster : 0);
        }
        const unsigned ballot = __ballot_sync(0xffffffffu, act);
        if (act) list[cnt + __popc(ballot & ((1u << lane) - 1u))] = entry;
        cnt += __popc(ballot);
      }
      if (lane == 0) list_count[buf] = cnt;
      __syncwarp();
      mbar_arrive(list_full(buf));
    }
    __syncwarp();
  }
  } else {
    if constexpr (D == 128 && !kMaskFast) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
    } else if constexpr (kPersist) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 192;" ::: "memory");
    }
    // ------------------------------------------------------------ softmax
    const int qi = warp >> 2;                       // which Q tile
    const int r = ((warp & 3) << 5) + lane;         // row in the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kTmemS + 128u * qi;
    const uint32_t tO = tmem + lane_off + C::kTmemO + uint32_t(D) * qi;
    const uint32_t tP = tmem + lane_off + C::kTmemP + C::kPStride * qi;
    const float c = p.c;
    const bool ragged_kv = (p.S_kv % kBN) != 0;
    // masked key tiles: their keys' ids or coordinates, staged per warp
    int32_t* kinfo = reinterpret_cast<int32_t*>(smem + C::kOffKinfo) + warp * kBN;
    int T = 0;      // key tiles done by this CTA, over all units (barrier parities)
    bool ok = true;
    for (int u = blockIdx.x, k = 0; ok && u < u_end; u += u_step, ++k) {
      const int* list;
      int n_list;
      ok = wait_list(k, &list, &n_list);
      if (!ok) break;
      const Unit x = decode_unit(p, u);
      const int bh = x.b * p.H + x.h;
      const int pair = x.pair;
      const int row = pair * 2 * kBM + qi * kBM + r;
      const bool row_valid = row < p.S_q;
      // Values only masked tiles use (the row's id or coordinate, the keys'
      // ids or coordinates) are read where they are used, from x.b and row,
      // so that nothing more stays live across the tile loop.
      int4 my_qs;
      make_walk(p, x.b, pair, qi, &my_qs);
      const UnitSched sched = unit_sched(p, x, list, n_list);
      // window variant: the row's window starts, once per unit (masks of
      // key tiles in raster order are built from them and the tile index)
      int ws0 = 0, ws1 = 0, ws2 = 0;
      if (kMaskFast && has_win) {
        const uint32_t qc =
            row_valid ? uint32_t(__ldg(p.coord_q + static_cast<int64_t>(x.b) * p.S_q + row)) : 0u;
        const WinRow wr = win_row(p, qc);
        ws0 = wr.s[0];
        ws1 = wr.s[1];
        ws2 = wr.s[2];
      }

      float m_run = -INFINITY;   // running max of scale*log2(e)*s, the offset of P
      float l_run = 0.f;         // running sum of P (fp32, before bf16 rounding)
      int lt = 0;                // tiles of this unit done
      int t = sched.t0;
      for (int j = sched.tile(t, t - 1); j < sched.n_kv; ++t, ++lt, ++T, j = sched.tile(t, j)) {
        bool masked;
        bool raster = false;   // window variant: a key tile in raster order
        if (list != nullptr) {
          masked = (list[t] >> (30 + qi)) & 1;
          raster = kMaskFast && (list[t] & kListRaster) != 0;
        } else {
          masked = (ragged_kv && j == p.n_kv_tiles - 1) || causal_partial(p, pair, qi, j) || has_win;
          if (has_seg) {
            const int4 ks = __ldg(sched.walk.kv_sum + j);
            masked = masked || !(my_qs.z && ks.z && my_qs.x == ks.x);
          }
        }
        const bool slow = masked || !(c > 0.f);
        // A masked tile's key ids / coordinates: loads issued before the wait
        // for S, so their latency hides behind it (warp-uniform: masked is the
        // same for every row of a Q tile).
        int32_t pre[4] = {0, 0, 0, 0};
        if (masked && has_sum && !raster) {
          // the keys' ids or coordinates (tile summaries come with one or the other)
          const int32_t* src = (has_win ? p.coord_kv : p.seg_kv) + static_cast<int64_t>(x.b) * p.S_kv;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int xk = j * kBN + lane + 32 * m;
            if (xk < p.S_kv) pre[m] = __ldg(src + xk);
          }
        }
        // visible keys of this row: all of an unmasked tile; a masked tile's
        // mask is built from the slot, in the window variant before the wait
        // for S, elsewhere where it is used (the exact paths)
        auto build_mask = [&](uint32_t (&mb)[4]) {
          const int j0 = j * kBN;
          const int n_valid = min(kBN, p.S_kv - j0);
          const int n_lim =
              p.causal ? max(0, min(n_valid, row + p.causal_off - j0 + 1)) : n_valid;
          const int64_t qrow = static_cast<int64_t>(x.b) * p.S_q + row;
          const int my_seg = (has_seg && row_valid) ? __ldg(p.seg_q + qrow) : 0;
          const uint32_t my_coord = (has_win && row_valid) ? uint32_t(__ldg(p.coord_q + qrow)) : 0u;
          const WinRow wr = win_row(p, my_coord);
          __syncwarp();
          const int mode = has_win ? 2 : (has_seg ? 1 : 0);
          const uint4 m =
              kMaskFast ? tile_mask(kinfo, mode, my_seg, wr.s[0], wr.s[1], wr.s[2], p.win_size[0],
                                    p.win_size[1], p.win_size[2], n_lim)
                        : tile_mask_call(kinfo, mode, my_seg, wr.s[0], wr.s[1], wr.s[2],
                                         p.win_size[0], p.win_size[1], p.win_size[2], n_lim);
          __syncwarp();   // every lane has read the slot before it is refilled
          mb[0] = m.x;
          mb[1] = m.y;
          mb[2] = m.z;
          mb[3] = m.w;
        };
        // Window variant: building the mask before the wait for S overlaps
        // it with the tensor core's Q K^T (measured +3 % on a 480p windowed
        // call) instead of putting it on the chain after S; the slot is
        // free, as the previous masked tile's mask was built before its
        // __syncwarp.  A key tile in raster order needs no slot: its mask
        // comes from the tile index.  The exact paths use this mask.
        uint32_t mb_early[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
        bool have_mask = false;
        if (kMaskFast && masked && has_sum) {
          if (raster) {
            const int j0 = j * kBN;
            const int n_valid = min(kBN, p.S_kv - j0);
            const int n_lim =
                p.causal ? max(0, min(n_valid, row + p.causal_off - j0 + 1)) : n_valid;
            const uint4 mk = raster_mask(p, j, n_lim, ws0, ws1, ws2);
            mb_early[0] = mk.x;
            mb_early[1] = mk.y;
            mb_early[2] = mk.z;
            mb_early[3] = mk.w;
          } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) kinfo[lane + 32 * m] = pre[m];
            build_mask(mb_early);
          }
          have_mask = true;
        }
        VIDATTN_TR(1 + qi, T, 0);
        ok = warp_wait_phase(s_full(qi), uint32_t(T) & 1u, abort_flag, p.err);
        VIDATTN_TR(1 + qi, T, 1);
        if (!ok) break;
        tc_fence_after();
        if (masked && has_sum && !have_mask) {
          // the previous masked tile's mask was built before this point (the
          // __syncwarp after it), so the slot is free
#pragma unroll
          for (int m = 0; m < 4; ++m) kinfo[lane + 32 * m] = pre[m];
        }

        if constexpr (C::kSepP) {
          // S row into registers; S's columns go back to the MMA warp once
          // this tile's P is computed (P has columns of its own).
          float s[kBN];
          load_s_row(tS, s);
          VIDATTN_TR(1 + qi, T, 2);
          uint32_t pk[2][32];
          float rs = 0.f, alpha = 1.f;
          bool rescale = false;
          // running-offset path first (see the aliased-P branch below); its
          // exponentials consume the S registers as they go, so the exact
          // path reads S from tensor memory again (still intact: s_free
          // comes after)
          bool exact = __any_sync(0xffffffffu, slow || (m_run == -INFINITY));
          if (!exact) {
            rs = exp_tile<kEmu>(s, c, m_run, pk);
            exact = __any_sync(0xffffffffu, !(rs <= kStaleSumLimit));
          }
          if (exact) {
            // the mask first: no S register is live across its call
            uint32_t mb[4] = {mb_early[0], mb_early[1], mb_early[2], mb_early[3]};
            if (masked && !have_mask) build_mask(mb);
            load_s_row(tS, s);
            float tile_max;
            if (!slow) {
              tile_max = row_max(s) * c;
            } else {
              float mx = -INFINITY;
#pragma unroll
              for (int xk = 0; xk < kBN; ++xk) {
                const bool valid = (mb[xk >> 5] >> (xk & 31)) & 1u;
                s[xk] = valid ? s[xk] * c : -INFINITY;
                mx = fmaxf(mx, s[xk]);
              }
              tile_max = mx;
            }
            const float m_new = fmaxf(m_run, tile_max);
            rescale = (m_new - m_run) > kRescaleThreshold;
            if (rescale) {
              alpha = ex2(m_run - m_new);
              m_run = m_new;
            }
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            if (!slow) {
              rs = exp_tile<kEmu>(s, c, msub, pk);
            } else {
              float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int xk = 0; xk < kBN; xk += 2) {
                const float e0 = ex2(s[xk] - msub);
                const float e1 = ex2(s[xk + 1] - msub);
                r4[(xk >> 1) & 3] += e0 + e1;
                pk[xk >> 6][(xk >> 1) & 31] = pack_bf16x2(e0, e1);
              }
              rs = (r4[0] + r4[1]) + (r4[2] + r4[3]);
            }
          }
          tc_fence_before();
          mbar_arrive(s_free(qi));
          l_run = l_run * alpha + rs;
          VIDATTN_TR(1 + qi, T, 3);
          // The previous P V of this tile has read P's columns and finished
          // accumulating O: P may be overwritten and O rescaled.  (Before a
          // unit's first tile the previous unit's epilogue waited for it.)
          if (lt > 0) {
            ok = warp_wait_phase(o_full(qi), uint32_t(T - 1) & 1u, abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
          }
          VIDATTN_TR(1 + qi, T, 4);
          tmem_st32(tP, pk[0]);
          tmem_st32(tP + 32, pk[1]);
          if (__any_sync(0xffffffffu, rescale && lt > 0)) {
#pragma unroll 1
            for (int kk = 0; kk < D / 32; ++kk) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * kk, o);
              tmem_ld_wait();
              reg_fence(o);
#pragma unroll
              for (int xk = 0; xk < 32; ++xk)
                o[xk] = __float_as_uint(__uint_as_float(o[xk]) * alpha);
              tmem_st32(tO + 32 * kk, o);
            }
          }
          tmem_st_wait();
        } else {
          // P = 2^(c*s - m_run) for this tile, rounded to bf16 into pk; rs = its
          // row sum in fp32.  Softmax does not depend on the offset m_run, so after
          // a row's first tile the running offset is used as it stands ("stale"
          // path, no max).  The offset only has to keep every exponential finite:
          // if the tile's sum exceeds 2^32 the row takes the exact path instead,
          // which computes the tile max, moves m_run up (rescaling O and l), and
          // redoes the exponentials.  The exact path also serves masked tiles,
          // a row's first tile, and scale <= 0.
          float rs = 0.f, alpha = 1.f;
          bool rescale = false;
          // warp-uniform choice: the stale path only if every row of the warp
          // can take it (with kMaskFast masked tiles too: hidden keys get p = 0)
          bool exact =
              __any_sync(0xffffffffu, (kMaskFast ? !(c > 0.f) : slow) || (m_run == -INFINITY));
          if (!exact) {
            // a masked tile: its mask first (before S occupies the registers),
            // then hidden keys' scores become -inf, i.e. p = 0 (the FMA-pipe
            // exponential clamps at 2^-125, far below bf16 P's resolution
            // against the row sum, which includes the row's running maximum)
            uint32_t mb[4] = {mb_early[0], mb_early[1], mb_early[2], mb_early[3]};
            if (kMaskFast && masked && !have_mask) build_mask(mb);
            float s[kBN];
            uint32_t pk[2][32];
            load_s_row(tS, s);
            VIDATTN_TR(1 + qi, T, 2);
            if (kMaskFast && masked) {
              // 32-key chunks that no row of the warp sees (a window's rows
              // often miss whole (t, h) rows of the tile) skip their
              // exponentials: p = 0 there (warp-uniform, no divergence)
              rs = 0.f;
#define VIDATTN_CHUNK(K)                                                         \
  if (__any_sync(0xffffffffu, mb[K] != 0u)) {                                    \
    rs += exp_chunk_masked<kEmu, 32 * K>(s, c, m_run, mb[K], pk);                \
  } else {                                                                       \
    _Pragma("unroll") for (int xk = 0; xk < 16; ++xk) pk[K >> 1][16 * (K & 1) + xk] = 0u; \
  }
              VIDATTN_CHUNK(0)
              VIDATTN_CHUNK(1)
              VIDATTN_CHUNK(2)
              VIDATTN_CHUNK(3)
#undef VIDATTN_CHUNK
            } else {
              rs = exp_tile<kEmu>(s, c, m_run, pk);
            }
            VIDATTN_TR(1 + qi, T, 3);
            exact = __any_sync(0xffffffffu, !(rs <= kStaleSumLimit));
            if (!exact) {
              tmem_st32(tS, pk[0]);
              tmem_st32(tS + 32, pk[1]);
            }
          }
          if (exact) {
            // Two passes over the tile, 32 columns at a time, straight from
            // tensor memory (S is intact: no P has been written yet).  The sum
            // restarts: a failed running-offset attempt leaves its sum in rs.
            rs = 0.f;
            uint32_t mb[4] = {mb_early[0], mb_early[1], mb_early[2], mb_early[3]};
            if (masked && !have_mask) build_mask(mb);
            // this chunk's 32 mask bits (kk is a runtime index: select, don't index)
            auto chunk_bits = [&](int kk) {
              return kk == 0 ? mb[0] : (kk == 1 ? mb[1] : (kk == 2 ? mb[2] : mb[3]));
            };
            float mx = -INFINITY;
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk) {
              uint32_t rr[32];
              tmem_ld32(tS + 32 * kk, rr);
              const uint32_t mk = chunk_bits(kk);
              tmem_ld_wait();
              reg_fence(rr);
#pragma unroll
              for (int xk = 0; xk < 32; ++xk)
                mx = fmaxf(mx, ((mk >> xk) & 1u) ? __uint_as_float(rr[xk]) * c : -INFINITY);
            }
            const float m_new = fmaxf(m_run, mx);
            rescale = (m_new - m_run) > kRescaleThreshold;   // false for -inf - -inf
            if (rescale) {
              alpha = ex2(m_run - m_new);   // 0 when m_run is -inf
              m_run = m_new;
            }
            const float msub = (m_run == -INFINITY) ? 0.f : m_run;
            // P chunk kk (keys 32kk..32kk+31) lands in columns [16kk, 16kk+16),
            // which hold S columns already read: chunks are processed in order.
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk) {
              uint32_t rr[32], wv[16];
              tmem_ld32(tS + 32 * kk, rr);
              const uint32_t mk = chunk_bits(kk);
              tmem_ld_wait();
              reg_fence(rr);
#pragma unroll
              for (int xk = 0; xk < 32; xk += 2) {
                const float e0 = ((mk >> xk) & 1u) ? ex2(__uint_as_float(rr[xk]) * c - msub) : 0.f;
                const float e1 =
                    ((mk >> (xk + 1)) & 1u) ? ex2(__uint_as_float(rr[xk + 1]) * c - msub) : 0.f;
                rs += e0 + e1;
                wv[xk >> 1] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tS + 16 * kk, wv);
            }
          }
          l_run = l_run * alpha + rs;
          tmem_st_wait();
          // Rescale this tile's O rows before the next P.V accumulates into them.
          if (__any_sync(0xffffffffu, rescale && lt > 0)) {
            ok = warp_wait_phase(o_full(qi), uint32_t(T - 1) & 1u, abort_flag, p.err);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int kk = 0; kk < D / 32; ++kk) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * kk, o);
              tmem_ld_wait();
              reg_fence(o);
#pragma unroll
              for (int xk = 0; xk < 32; ++xk)
                o[xk] = __float_as_uint(__uint_as_float(o[xk]) * alpha);
              tmem_st32(tO + 32 * kk, o);
            }
            tmem_st_wait();
          }
        }
        tc_fence_before();
        mbar_arrive(p_full(qi));
        VIDATTN_TR(1 + qi, T, 5);
      }
      if (!ok) break;
      release_list(k);

      // ---------------------------------------------------------- epilogue
      // O of the unit's last tile is complete once its P V has run.  The
      // next unit's first P V overwrites O only after this warpgroup's
      // p_full arrival for that tile, which follows these reads.
      if (lt > 0) {
        ok = warp_wait_phase(o_full(qi), uint32_t(T - 1) & 1u, abort_flag, p.err);
        if (!ok) break;
        tc_fence_after();
      }
      const bool empty = !(l_run > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l_run;
      const float lse_row = empty ? -INFINITY : (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      if constexpr (!kSplit) {
        const int64_t orow = static_cast<int64_t>(bh) * p.S_q + row;
        uint16_t* out_row = p.out + orow * D;
#pragma unroll 1
        for (int kk = 0; kk < D / 32; ++kk) {
          uint32_t o[32];
          if (lt > 0) {
            tmem_ld32(tO + 32 * kk, o);
            tmem_ld_wait();
            reg_fence(o);
          } else {
#pragma unroll
            for (int xk = 0; xk < 32; ++xk) o[xk] = 0u;
          }
          uint32_t wv[16];
#pragma unroll
          for (int xk = 0; xk < 16; ++xk)
            wv[xk] = pack_bf16x2(__uint_as_float(o[2 * xk]) * inv_l,
                                 __uint_as_float(o[2 * xk + 1]) * inv_l);
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(out_row + 32 * kk);
#pragma unroll
            for (int xk = 0; xk < 4; ++xk)
              dst[xk] = make_uint4(wv[4 * xk], wv[4 * xk + 1], wv[4 * xk + 2], wv[4 * xk + 3]);
          }
        }
        if (row_valid) p.lse[orow] = lse_row;
      } else {
        // one key split of the row: O / l and the split's log-sum-exp in
        // fp32, merged by split_combine_kernel
        const int64_t prow = (static_cast<int64_t>(bh) * p.n_split + x.split) * p.S_q + row;
        float* po = p.part_o + prow * D;
#pragma unroll 1
        for (int kk = 0; kk < D / 32; ++kk) {
          uint32_t o[32];
          if (lt > 0) {
            tmem_ld32(tO + 32 * kk, o);
            tmem_ld_wait();
            reg_fence(o);
          } else {
#pragma unroll
            for (int xk = 0; xk < 32; ++xk) o[xk] = 0u;
          }
          if (row_valid) {
            float4* dst = reinterpret_cast<float4*>(po + 32 * kk);
#pragma unroll
            for (int xk = 0; xk < 8; ++xk)
              dst[xk] = make_float4(__uint_as_float(o[4 * xk]) * inv_l,
                                    __uint_as_float(o[4 * xk + 1]) * inv_l,
                                    __uint_as_float(o[4 * xk + 2]) * inv_l,
                                    __uint_as_float(o[4 * xk + 3]) * inv_l);
          }
        }
        if (row_valid) p.part_lse[prow] = lse_row;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Merges the key splits of a split launch: per query row, with lse_s and
// O_s (O / l) of each split s, lse = log sum_s exp(lse_s) and
// out = sum_s exp(lse_s - lse) O_s, rounded once to bf16.  A row no split
// saw (every lse_s = -inf) gets out = 0, lse = -inf.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256) split_combine_kernel(const float* __restrict__ part_o,
                                                            const float* __restrict__ part_lse,
                                                            uint16_t* __restrict__ out,
                                                            float* __restrict__ lse, int S_q,
                                                            int n_split, int64_t n_rows) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n_rows) return;
  const int64_t bh = w / S_q;
  const int64_t row = w - bh * S_q;
  constexpr int kPer = D / 32;   // columns per lane
  float mx = -INFINITY;
  for (int s = 0; s < n_split; ++s)
    mx = fmaxf(mx, __ldg(part_lse + (bh * n_split + s) * S_q + row));
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float total = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < n_split; ++s) {
      const int64_t prow = (bh * n_split + s) * S_q + row;
      const float ls = __ldg(part_lse + prow);
      if (ls == -INFINITY) continue;
      const float wgt = exp2f((ls - mx) * 1.44269504088896341f);
      total += wgt;
      const float* po = part_o + prow * D + lane * kPer;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += wgt * __ldg(po + e);
    }
  }
  const float inv = total > 0.f ? 1.f / total : 0.f;
  uint16_t* orow = out + w * D + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; e += 2) {
    const uint32_t pk = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    *reinterpret_cast<uint32_t*>(orow + e) = pk;
  }
  if (lane == 0) lse[w] = total > 0.f ? mx + __logf(total) : -INFINITY;
}

}  // namespace vidattn
