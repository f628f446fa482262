// Host side of the vidattn C ABI: argument checks, TMA descriptors, the
// tile-summary scratch cache, kernel launches (attention, causal and window
// variants, tile summaries, the rotary embedding), and the host-buffer entry
// point's copy pipeline.  The operations and the argument contracts are
// documented in include/vidattn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "../../include/vidattn.h"
#include "classify.cuh"
#include "fwd_kernel.cuh"
#include "rope3d.cuh"

namespace vidattn {

#ifdef VIDATTN_TRACE
// Trace builds only: the buffer vidattn_trace_set() names (4 x 64 x 16 u64).
unsigned long long* g_trace = nullptr;
#endif

// Device error word: kernels OR error bits into it (see kErrTimeout).
__device__ int g_device_error = 0;

// Scratch of vidattn_fwd_noalloc: the per-tile segment summaries (one int4
// per 128 tokens of seg_q and of seg_kv, per batch entry) live in this fixed
// array instead of memory the library allocates.  Every GPU that loads the
// library holds it (512 KiB) until the process exits.  Host code must not
// pass the symbol itself to a kernel: in host code it names a host-side
// stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (see noalloc_scratch below).
constexpr size_t kNoAllocMaxTiles = 32768;
static __device__ __align__(256) int4 g_noalloc_summaries[kNoAllocMaxTiles];

namespace {

constexpr const char* kVersion = "vidattn 0.2 (sm_100a: TMA + tcgen05/TMEM, persistent)";

// Split heuristic: a launch with fewer than kSplitFillSMs / 2 work units
// (256-row query blocks x heads x batch) splits each block's key tiles into
// up to kMaxAutoSplit ranges, enough to give about kSplitFillSMs units (the
// B200's 148 SMs), at least kMinSplitTiles key tiles per split: below that
// the merge kernel and each split's own first tile (two passes) cost more
// than the parallelism gains (measured: the 512-token tiny workload takes
// 16.7 us unsplit, 19.6 us in 2 splits, 18.2 us in 4).
constexpr int kSplitFillSMs = 148;
constexpr int kMaxAutoSplit = 16;
constexpr int kMinSplitTiles = 8;
// Persistent grid only for units of at most this many key tiles (below).
constexpr int kPersistMaxTiles = 64;
constexpr int kMaxSplit = 64;   // largest VIDATTN_SPLIT_KV request

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// bf16 [BH, S, D] as a 3-D tensor map {D, S, BH}; box {64, 128, 1}, 128-byte
// swizzle.  Rows past S read as zeros.
bool encode_bhsd(CUtensorMap* map, const void* ptr, int64_t BH, int64_t S, int D) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(S > 0 ? S : 1), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(D) * 2 * cuuint64_t(S > 0 ? S : 1)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                   strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  uint32_t attrs_set = 0;   // bit (kernel variant index) once its smem limit is raised
  int* err = nullptr;       // device address of g_device_error on this device
  int rope_grid[4] = {};    // persistent grid of each rope3d variant (SMs x resident CTAs)
  int sms = 0;              // streaming multiprocessors (the attention kernel's grid bound)
  // vidattn_fwd_host's copy streams (host-to-device, device-to-host) and
  // its second compute stream
  cudaStream_t copy_in = nullptr, copy_out = nullptr, compute2 = nullptr;
};

// Recently encoded tensor maps (per device): a call on the same buffers and
// shape reuses them instead of encoding three descriptors again.
struct MapKey {
  int dev;
  const void* ptr;
  int64_t BH, S;
  int D;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && ptr == o.ptr && BH == o.BH && S == o.S && D == o.D;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  uint64_t stamp;
};
constexpr int kMapCacheSize = 16;
MapEntry g_map_cache[kMapCacheSize];
int g_map_used = 0;
uint64_t g_map_clock = 0;
std::mutex g_map_mu;

using FwdKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const FwdParams);
// Variants of the attention kernel.  One CTA per unit, keys not split (the
// common launch): head dim x exponentials per 16 keys on the FMA pipe.
constexpr int kEmuChoices[] = {0, 2, 4, 6, 8};
constexpr int kNumEmu = 5;
template <int D>
FwdKernel fwd_variant(int e) {
  switch (e) {
    case 0: return vidattn_fwd_kernel<D, 0, false, false, false>;
    case 1: return vidattn_fwd_kernel<D, 2, false, false, false>;
    case 2: return vidattn_fwd_kernel<D, 4, false, false, false>;
    case 3: return vidattn_fwd_kernel<D, 6, false, false, false>;
    default: return vidattn_fwd_kernel<D, 8, false, false, false>;
  }
}
// Persistent or split launches: the head dim's default share (4 of 16 at
// D = 128, 2 of 16 at D = 64); a split launch is never persistent (it has
// fewer units than SMs).
FwdKernel fwd_persist_variant(int D) {
  return D == 128 ? vidattn_fwd_kernel<128, 4, false, true, false>
                  : vidattn_fwd_kernel<64, 2, false, true, false>;
}
FwdKernel fwd_split_variant(int D) {
  return D == 128 ? vidattn_fwd_kernel<128, 4, false, false, true>
                  : vidattn_fwd_kernel<64, 2, false, false, true>;
}
// 3D neighbourhood windows: masked tiles on the running-offset path (D = 128,
// 2 of 16 exponentials on the FMA pipe: the mask work takes issue slots, and
// 2 measured 3 % faster than 4 on the 11^3 window over the 480p volume);
// D = 64 uses the default kernel.  Never persistent (a window call's units
// span the whole key range of its tile summaries).
FwdKernel fwd_window_variant(int D, bool split) {
  if (split)
    return D == 128 ? vidattn_fwd_kernel<128, 2, true, false, true>
                    : vidattn_fwd_kernel<64, 2, false, false, true>;
  return D == 128 ? vidattn_fwd_kernel<128, 2, true, false, false>
                  : vidattn_fwd_kernel<64, 2, false, false, false>;
}
// Default share of exponentials moved off the MUFU unit (measured best on
// B200: 4 of 16 at D = 128, 2 of 16 at D = 64, where the FMA-pipe version's
// extra instructions cost more than the MUFU time they save).
// VIDATTN_EMU (0, 2, 4, 6 or 8 per 16 keys) overrides, for experiments.
int emu_index(int D) {
  static const int forced = [] {
    const char* e = getenv("VIDATTN_EMU");
    if (!e) return -1;
    const int v = atoi(e);
    for (int i = 0; i < kNumEmu; ++i)
      if (kEmuChoices[i] == v) return i;
    return -1;
  }();
  if (forced >= 0) return forced;
  return D == 128 ? 2 : 1;
}
std::mutex g_mu;
std::map<int, DeviceInfo> g_devices;

struct Scratch {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::map<std::pair<int, cudaStream_t>, Scratch> g_scratch;

int ensure_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VIDATTN_ERR_CUDA;
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& info = g_devices[dev];
  if (!info.checked) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return VIDATTN_ERR_CUDA;
    info.checked = true;
    info.ok = (major == 10 && minor == 0);
    if (cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return VIDATTN_ERR_CUDA;
  }
  if (!info.ok) return VIDATTN_ERR_NO_DEVICE;
  if (info.err == nullptr) {
    void* e = nullptr;
    if (cudaGetSymbolAddress(&e, g_device_error) != cudaSuccess || e == nullptr)
      return VIDATTN_ERR_CUDA;
    info.err = static_cast<int*>(e);
  }
  if (info.attrs_set == 0) {
    auto smem = [](FwdKernel k, int bytes) {
      return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
             cudaSuccess;
    };
    bool ok = true;
    for (int e = 0; e < kNumEmu; ++e)
      ok = ok && smem(fwd_variant<64>(e), FwdCfg<64>::kSmemBytes) &&
           smem(fwd_variant<128>(e), FwdCfg<128>::kSmemBytes);
    for (int D : {64, 128}) {
      const int bytes = D == 128 ? FwdCfg<128>::kSmemBytes : FwdCfg<64>::kSmemBytes;
      ok = ok && smem(fwd_persist_variant(D), bytes) && smem(fwd_split_variant(D), bytes) &&
           smem(fwd_window_variant(D, false), bytes) && smem(fwd_window_variant(D, true), bytes);
    }
    if (!ok) return VIDATTN_ERR_CUDA;
    info.attrs_set = 1;
  }
  return VIDATTN_OK;
}

// Scratch of at least `bytes` for (dev, stream).  Growing synchronises the
// stream first, so a buffer still in use by earlier work is never freed.
void* scratch_for(int dev, cudaStream_t stream, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  Scratch& s = g_scratch[{dev, stream}];
  if (s.bytes >= bytes) return s.ptr;
  if (s.ptr) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return nullptr;
    cudaFree(s.ptr);
    s.ptr = nullptr;
    s.bytes = 0;
  }
  size_t want = bytes < 4096 ? 4096 : bytes;
  if (cudaMalloc(&s.ptr, want) != cudaSuccess) {
    s.ptr = nullptr;
    return nullptr;
  }
  s.bytes = want;
  return s.ptr;
}

// Device address of g_noalloc_summaries on `dev` (which must be current),
// looked up on the first call for that device and remembered.
std::map<int, int4*> g_noalloc_ptr;
int noalloc_scratch(int dev, int4** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_noalloc_ptr.find(dev);
  if (it == g_noalloc_ptr.end()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_summaries) != cudaSuccess || p == nullptr)
      return VIDATTN_ERR_CUDA;
    it = g_noalloc_ptr.emplace(dev, static_cast<int4*>(p)).first;
  }
  *out = it->second;
  return VIDATTN_OK;
}

int* device_error_word(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_devices[dev].err;
}

int device_sms(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_devices[dev].sms;
}

// Tensor map of bf16 [BH, S, D] at ptr on dev, from the cache when present.
bool cached_map(int dev, const void* ptr, int64_t BH, int64_t S, int D, CUtensorMap* out) {
  const MapKey key{dev, ptr, BH, S, D};
  std::lock_guard<std::mutex> lk(g_map_mu);
  for (int i = 0; i < g_map_used; ++i) {
    if (g_map_cache[i].key == key) {
      g_map_cache[i].stamp = ++g_map_clock;
      *out = g_map_cache[i].map;
      return true;
    }
  }
  if (!encode_bhsd(out, ptr, BH, S, D)) return false;
  int slot = g_map_used;
  if (g_map_used < kMapCacheSize) {
    ++g_map_used;
  } else {
    slot = 0;
    for (int i = 1; i < kMapCacheSize; ++i)
      if (g_map_cache[i].stamp < g_map_cache[slot].stamp) slot = i;
  }
  g_map_cache[slot] = MapEntry{key, *out, ++g_map_clock};
  return true;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

int check_args(const void* q, const void* k, const void* v, const int32_t* seg_q,
               const int32_t* seg_kv, const void* out, const float* lse, int B, int H, int S_q,
               int S_kv, int D) {
  if (S_q > 0 && (!q || !out || !lse)) return VIDATTN_ERR_NULL;
  if (S_kv > 0 && (!k || !v)) return VIDATTN_ERR_NULL;
  if ((seg_q == nullptr) != (seg_kv == nullptr)) return VIDATTN_ERR_SEG_PAIR;
  if (D != 64 && D != 128) return VIDATTN_ERR_UNSUPPORTED_D;
  if (B < 1 || H < 1 || B > 65535 || H > 65535 || S_q < 0 || S_kv < 0)
    return VIDATTN_ERR_BAD_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(lse, 4) || (seg_q && (!aligned(seg_q, 4) || !aligned(seg_kv, 4))))
    return VIDATTN_ERR_MISALIGNED;
  return VIDATTN_OK;
}

// A 3D neighbourhood window for launch_fwd.
struct WinSpec {
  const int32_t* coord_q;
  const int32_t* coord_kv;
  int size[3], extent[3], clamped;
};

// Bytes of split partials (O / l and lse per row and split, fp32) for a launch.
size_t split_bytes(int B, int H, int S_q, int D, int n_split) {
  if (n_split <= 1) return 0;
  return size_t(B) * H * n_split * S_q * (size_t(D) + 1) * 4;
}

// The launch's key splits: `requested` when the caller asks for a number
// (VIDATTN_SPLIT_KV), else the heuristic of vidattn_split_count.
int choose_split(int B, int H, int S_q, int S_kv, bool global_walk, int requested) {
  if (S_q <= 0 || S_kv <= 0 || global_walk) return 1;
  if (requested > 0) return requested;
  const int64_t units = int64_t(B) * H * ((S_q + 2 * kBM - 1) / (2 * kBM));
  if (units * 2 >= kSplitFillSMs) return 1;
  const int n_kv = (S_kv + kBN - 1) / kBN;
  int64_t want = (kSplitFillSMs + units - 1) / units;
  if (want > n_kv / kMinSplitTiles) want = n_kv / kMinSplitTiles;
  if (want > kMaxAutoSplit) want = kMaxAutoSplit;
  return want < 1 ? 1 : int(want);
}

// Persistent grid or one CTA per unit (unsplit launches).  Persistence
// overlaps a unit's epilogue with the next unit's loads and first Q K^T,
// which pays when units are short: measured at D = 128 with more units than
// SMs, +13 % at 4 key tiles per unit, +9 % at 8, +6 % at 16, +3 % at 32,
// +1 % at 64; at D = 64 (16 tiles) nothing.  On long units the hardware's
// dynamic placement of one CTA per unit balances the SMs better than the
// static round-robin (the 480p and 720p workloads lose 1-2 % persistent).
// VIDATTN_PERSIST=0/1 overrides, for experiments.
bool use_persistent(int64_t n_units, int sms, int n_kv_tiles, int D) {
  static const int forced = [] {
    const char* e = getenv("VIDATTN_PERSIST");
    return e ? (atoi(e) != 0 ? 1 : 0) : -1;
  }();
  if (forced >= 0) return forced == 1;
  return D == 128 && n_units > sms && n_kv_tiles <= kPersistMaxTiles;
}

// CTAs of the attention launch: one per unit, or persistent with one per SM.
int launch_grid(int64_t n_units, int sms, bool persist) {
  return int(persist ? (n_units > sms ? sms : n_units) : n_units);
}

template <int D>
int launch_fwd(int dev, const void* q, const void* k, const void* v, const int32_t* seg_q,
               const int32_t* seg_kv, const int4* q_sum, const int4* kv_sum, void* out,
               float* lse, int B, int H, int S_q, int S_kv, float scale, cudaStream_t stream,
               int flags = 0, const WinSpec* win = nullptr, int n_split = 1,
               float* part = nullptr) {
  CUtensorMap tq, tk, tv;
  const int64_t BH = int64_t(B) * H;
  // With no keys the K/V maps are never read; they are encoded over q.
  const void* kp = S_kv > 0 ? k : q;
  const void* vp = S_kv > 0 ? v : q;
  if (!cached_map(dev, q, BH, S_q, D, &tq) || !cached_map(dev, kp, BH, S_kv, D, &tk) ||
      !cached_map(dev, vp, BH, S_kv, D, &tv))
    return VIDATTN_ERR_CUDA;
  FwdParams p{};
  p.seg_q = seg_q;
  p.seg_kv = seg_kv;
  p.q_sum = q_sum;
  p.kv_sum = kv_sum;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.err = device_error_word(dev);
  p.H = H;
  p.S_q = S_q;
  p.S_kv = S_kv;
  p.n_q_tiles = (S_q + kBM - 1) / kBM;
  p.n_kv_tiles = (S_kv + kBN - 1) / kBN;
  p.causal = (flags & VIDATTN_CAUSAL) ? 1 : 0;
  p.causal_off = S_kv - S_q;
  p.n_pairs = (S_q + 2 * kBM - 1) / (2 * kBM);
  p.n_split = n_split;
  const int64_t n_units = int64_t(B) * H * p.n_pairs * n_split;
  if (n_units > INT_MAX) return VIDATTN_ERR_BAD_SHAPE;
  p.n_units = int(n_units);
  if (n_split > 1) {
    p.part_o = part;
    p.part_lse = part + size_t(B) * H * n_split * S_q * D;
  }
  if (win) {
    p.coord_q = win->coord_q;
    p.coord_kv = win->coord_kv;
    for (int a = 0; a < 3; ++a) {
      p.win_size[a] = win->size[a];
      p.win_extent[a] = win->extent[a];
    }
    p.win_clamped = win->clamped;
    p.div_wg = make_fastdiv(uint32_t(win->extent[2]));
    p.div_hg = make_fastdiv(uint32_t(win->extent[1]));
  }
  p.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
#ifdef VIDATTN_TRACE
  p.trace = g_trace;
#endif
  // persistent: at most one CTA per SM (tensor and shared memory are sized
  // for one), each looping over units; else one CTA per unit
  const int sms = device_sms(dev);
  const bool persist = !win && n_split == 1 && use_persistent(n_units, sms, p.n_kv_tiles, D);
  const int grid = launch_grid(n_units, sms, persist);
  FwdKernel kernel = win ? fwd_window_variant(D, n_split > 1)
                         : (n_split > 1 ? fwd_split_variant(D)
                                        : (persist ? fwd_persist_variant(D)
                                                   : fwd_variant<D>(emu_index(D))));
  kernel<<<grid, kFwdThreads, FwdCfg<D>::kSmemBytes, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return VIDATTN_ERR_CUDA;
  if (n_split > 1) {
    const int64_t rows = int64_t(B) * H * S_q;
    const int64_t blocks = (rows + 7) / 8;   // 8 warps, one row each
    split_combine_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
        p.part_o, p.part_lse, static_cast<uint16_t*>(out), lse, S_q, n_split, rows);
    if (cudaGetLastError() != cudaSuccess) return VIDATTN_ERR_CUDA;
  }
  return VIDATTN_OK;
}

// The streams of vidattn_fwd_host on device dev (created on first use).
bool host_streams(int dev, cudaStream_t* in, cudaStream_t* out, cudaStream_t* comp2) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& info = g_devices[dev];
  for (cudaStream_t* sp : {&info.copy_in, &info.copy_out, &info.compute2})
    if (!*sp && cudaStreamCreateWithFlags(sp, cudaStreamNonBlocking) != cudaSuccess) return false;
  *in = info.copy_in;
  *out = info.copy_out;
  *comp2 = info.compute2;
  return true;
}

// Below this many bytes of copies, vidattn_fwd_host does not split the work.
constexpr size_t kPipelineMinBytes = size_t(64) << 20;
constexpr int kPipelineChunks = 8;

// One warp waits on an mbarrier that nothing ever arrives on, through the
// attention kernel's bounded wait; it gives up after timeout_ns and reports.
__global__ void selftest_timeout_kernel(int* err, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  wait_phase(smem_u32(&bar), 0, &abort_flag, err, timeout_ns);
  __syncwarp();
}


using RopeKernel = void (*)(const RopeParams);
RopeKernel rope_variant(int i) {
  switch (i) {
    case 0: return rope3d_kernel<64, true>;
    case 1: return rope3d_kernel<64, false>;
    case 2: return rope3d_kernel<128, true>;
    default: return rope3d_kernel<128, false>;
  }
}

// SMs x resident CTAs of rope3d variant i on device dev (0 on failure).
int rope_grid(int dev, int i) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& info = g_devices[dev];
  if (info.rope_grid[i] == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rope_variant(i), kRopeThreads, 0) !=
            cudaSuccess)
      return 0;
    info.rope_grid[i] = sms * (per_sm > 0 ? per_sm : 1);
  }
  return info.rope_grid[i];
}

// Fills the per-column frequencies and the per-feature pairing tables.
void rope_tables(RopeParams& p, int D, const int bands[3], double theta, bool half_split) {
  int start = 0;
  for (int a = 0; a < 3; ++a) {
    const int d = bands[a], half = d / 2;
    for (int k = 0; k < half; ++k) {
      const int c = start / 2 + k;
      p.freq[c] = std::pow(theta, -2.0 * k / d);
      const int f0 = half_split ? start + k : start + 2 * k;
      const int f1 = half_split ? start + k + half : start + 2 * k + 1;
      p.col[f0] = p.col[f1] = static_cast<uint8_t>(c);
      p.partner[f0] = static_cast<uint8_t>(f1);
      p.partner[f1] = static_cast<uint8_t>(f0);
      p.first[f0] = 1;
      p.first[f1] = 0;
    }
    start += d;
  }
  (void)D;
}

}  // namespace
}  // namespace vidattn

using namespace vidattn;

extern "C" {

VIDATTN_API const char* vidattn_version(void) { return kVersion; }

VIDATTN_API const char* vidattn_status_string(int status) {
  switch (status) {
    case VIDATTN_OK: return "ok";
    case VIDATTN_ERR_NULL: return "a required pointer is NULL";
    case VIDATTN_ERR_UNSUPPORTED_D: return "head dim D must be 64 or 128";
    case VIDATTN_ERR_BAD_SHAPE: return "B, H, S_q or S_kv out of range";
    case VIDATTN_ERR_MISALIGNED: return "pointer misaligned (q/k/v/out need 16 bytes, lse/seg 4)";
    case VIDATTN_ERR_CUDA: return "CUDA error";
    case VIDATTN_ERR_TIMEOUT: return "a kernel wait timed out";
    case VIDATTN_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    case VIDATTN_ERR_SEG_PAIR: return "seg_q and seg_kv must both be NULL or both be set";
    case VIDATTN_ERR_SCRATCH_LIMIT:
      return "shape too large for vidattn_fwd_noalloc's fixed scratch: "
             "B*(ceil(S_q/128)+ceil(S_kv/128)) must be <= 32768";
    default: return "unknown status";
  }
}

VIDATTN_API int vidattn_split_count(const int32_t* seg_q, int B, int H, int S_q, int S_kv,
                                    int flags) {
  if (B < 1 || H < 1 || S_q < 1 || S_kv < 0) return 0;
  const int requested = (flags >> 8) & 0xFF;
  if (requested > kMaxSplit) return 0;
  const bool global_walk = seg_q != nullptr && (S_kv + kBN - 1) / kBN > kMaxListedTiles;
  return choose_split(B, H, S_q, S_kv, global_walk, requested);
}

VIDATTN_API int vidattn_launch_plan(const int32_t* seg_q, int B, int H, int S_q, int S_kv,
                                    int D, int flags, int* grid_ctas, int* key_splits,
                                    int* persistent) {
  if (!grid_ctas || !key_splits || !persistent) return VIDATTN_ERR_NULL;
  if (D != 64 && D != 128) return VIDATTN_ERR_UNSUPPORTED_D;
  if (flags & ~(VIDATTN_CAUSAL | VIDATTN_SPLIT_KV(0xFF))) return VIDATTN_ERR_BAD_SHAPE;
  const int n_split = vidattn_split_count(seg_q, B, H, S_q, S_kv, flags);
  if (n_split < 1) return VIDATTN_ERR_BAD_SHAPE;
  int dev = 0;
  const int st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;
  const int64_t n_units =
      int64_t(B) * H * ((S_q + 2 * kBM - 1) / (2 * kBM)) * n_split;
  if (n_units > INT_MAX) return VIDATTN_ERR_BAD_SHAPE;
  const int sms = device_sms(dev);
  const bool persist =
      n_split == 1 && use_persistent(n_units, sms, (S_kv + kBN - 1) / kBN, D);
  *grid_ctas = launch_grid(n_units, sms, persist);
  *key_splits = n_split;
  *persistent = persist ? 1 : 0;
  return VIDATTN_OK;
}

VIDATTN_API int vidattn_kernels_per_call(const int32_t* seg_q, const int32_t* seg_kv, int B,
                                         int H, int S_q, int S_kv, int D, int flags) {
  (void)seg_kv;
  (void)D;
  if (B < 1 || H < 1 || S_q < 1) return 0;
  const int n_split = vidattn_split_count(seg_q, B, H, S_q, S_kv, flags);
  return (seg_q ? 2 : 1) + (n_split > 1 ? 1 : 0);
}

VIDATTN_API int vidattn_fwd(const void* q, const void* k, const void* v, const int32_t* seg_q,
                            const int32_t* seg_kv, void* out, float* lse, int B, int H, int S_q,
                            int S_kv, int D, float scale, vidattn_stream_t stream_) {
  return vidattn_fwd_ex(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale, 0, stream_);
}

VIDATTN_API int vidattn_fwd_ex(const void* q, const void* k, const void* v,
                               const int32_t* seg_q, const int32_t* seg_kv, void* out, float* lse,
                               int B, int H, int S_q, int S_kv, int D, float scale, int flags,
                               vidattn_stream_t stream_) {
  if (flags & ~(VIDATTN_CAUSAL | VIDATTN_SPLIT_KV(0xFF))) return VIDATTN_ERR_BAD_SHAPE;
  if (((flags >> 8) & 0xFF) > kMaxSplit) return VIDATTN_ERR_BAD_SHAPE;
  int st = check_args(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D);
  if (st != VIDATTN_OK) return st;
  if (!std::isfinite(scale)) return VIDATTN_ERR_BAD_SHAPE;
  if (S_q == 0) return VIDATTN_OK;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev = 0;
  st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;

  // scratch: the segment summaries, then (split launches) the partials
  const int n_split = vidattn_split_count(seg_q, B, H, S_q, S_kv, flags);
  const int nq = (S_q + kSegTile - 1) / kSegTile;
  const int nk = (S_kv + kSegTile - 1) / kSegTile;
  const size_t sum_bytes =
      seg_q ? (sizeof(int4) * size_t(B) * (size_t(nq) + size_t(nk)) + 255) & ~size_t(255) : 0;
  const size_t part_bytes = split_bytes(B, H, S_q, D, n_split);
  char* buf = nullptr;
  if (sum_bytes + part_bytes > 0) {
    buf = static_cast<char*>(scratch_for(dev, stream, sum_bytes + part_bytes));
    if (!buf) return VIDATTN_ERR_CUDA;
  }
  const int4* q_sum = nullptr;
  const int4* kv_sum = nullptr;
  if (seg_q) {
    int4* sums = reinterpret_cast<int4*>(buf);
    q_sum = sums;
    kv_sum = sums + size_t(B) * nq;
    dim3 grid(nq > nk ? nq : nk, B, 2);
    seg_tile_classify_kernel<<<grid, 128, 0, stream>>>(seg_q, seg_kv, sums, sums + size_t(B) * nq,
                                                       S_q, S_kv);
    if (cudaGetLastError() != cudaSuccess) return VIDATTN_ERR_CUDA;
  }
  float* part = part_bytes ? reinterpret_cast<float*>(buf + sum_bytes) : nullptr;
  const int attn_flags = flags & VIDATTN_CAUSAL;
  if (D == 64)
    return launch_fwd<64>(dev, q, k, v, seg_q, seg_kv, q_sum, kv_sum, out, lse, B, H, S_q, S_kv,
                          scale, stream, attn_flags, nullptr, n_split, part);
  return launch_fwd<128>(dev, q, k, v, seg_q, seg_kv, q_sum, kv_sum, out, lse, B, H, S_q, S_kv,
                         scale, stream, attn_flags, nullptr, n_split, part);
}

VIDATTN_API int vidattn_fwd_window(const void* q, const void* k, const void* v,
                                   const int32_t* coord_q, const int32_t* coord_kv, void* out,
                                   float* lse, int B, int H, int S_q, int S_kv, int D,
                                   float scale, int win_t, int win_h, int win_w, int T, int Hg,
                                   int Wg, int flags, vidattn_stream_t stream_) {
  if (!coord_q || !coord_kv) return VIDATTN_ERR_NULL;
  if (flags & ~VIDATTN_WINDOW_CLAMPED) return VIDATTN_ERR_BAD_SHAPE;
  int st = check_args(q, k, v, coord_q, coord_kv, out, lse, B, H, S_q, S_kv, D);
  if (st != VIDATTN_OK) return st;
  if (!std::isfinite(scale)) return VIDATTN_ERR_BAD_SHAPE;
  const int size[3] = {win_t, win_h, win_w};
  const int extent[3] = {T, Hg, Wg};
  const int max_extent[3] = {1024, 2048, 2048};
  for (int a = 0; a < 3; ++a) {
    if (size[a] < 1 || size[a] % 2 == 0 || extent[a] < 1 || extent[a] > max_extent[a])
      return VIDATTN_ERR_BAD_SHAPE;
  }
  if (int64_t(S_kv) > int64_t(kMaxListedTiles) * kBN) return VIDATTN_ERR_BAD_SHAPE;
  if (S_q == 0) return VIDATTN_OK;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev = 0;
  st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;

  const int nq = (S_q + kSegTile - 1) / kSegTile;
  const int nk = (S_kv + kSegTile - 1) / kSegTile;
  const int n_split = choose_split(B, H, S_q, S_kv, false, 0);
  const size_t box_bytes =
      (sizeof(int4) * size_t(B) * (size_t(nq) + size_t(nk > 0 ? nk : 1)) + 255) & ~size_t(255);
  const size_t part_bytes = split_bytes(B, H, S_q, D, n_split);
  char* buf = static_cast<char*>(scratch_for(dev, stream, box_bytes + part_bytes));
  if (!buf) return VIDATTN_ERR_CUDA;
  int4* q_box = reinterpret_cast<int4*>(buf);
  int4* kv_box = q_box + size_t(B) * nq;
  dim3 grid(nq > nk ? nq : nk, B, 2);
  win_tile_bbox_kernel<<<grid, 128, 0, stream>>>(coord_q, coord_kv, q_box, kv_box, S_q, S_kv,
                                                  T, Hg, Wg);
  if (cudaGetLastError() != cudaSuccess) return VIDATTN_ERR_CUDA;
  WinSpec win{coord_q, coord_kv, {win_t, win_h, win_w}, {T, Hg, Wg},
              (flags & VIDATTN_WINDOW_CLAMPED) ? 1 : 0};
  float* part = part_bytes ? reinterpret_cast<float*>(buf + box_bytes) : nullptr;
  if (D == 64)
    return launch_fwd<64>(dev, q, k, v, nullptr, nullptr, q_box, kv_box, out, lse, B, H, S_q, S_kv,
                          scale, stream, 0, &win, n_split, part);
  return launch_fwd<128>(dev, q, k, v, nullptr, nullptr, q_box, kv_box, out, lse, B, H, S_q, S_kv,
                         scale, stream, 0, &win, n_split, part);
}

VIDATTN_API int vidattn_fwd_host(const void* h_q, const void* h_k, const void* h_v,
                                 const int32_t* h_seg_q, const int32_t* h_seg_kv, void* h_out,
                                 float* h_lse, void* d_q, void* d_k, void* d_v, int32_t* d_seg_q,
                                 int32_t* d_seg_kv, void* d_out, float* d_lse, int B, int H,
                                 int S_q, int S_kv, int D, float scale,
                                 vidattn_stream_t stream_) {
  if (!h_q || !h_k || !h_v || !h_out || !h_lse) return VIDATTN_ERR_NULL;
  if ((h_seg_q == nullptr) != (h_seg_kv == nullptr) ||
      (h_seg_q == nullptr) != (d_seg_q == nullptr) ||
      (d_seg_q == nullptr) != (d_seg_kv == nullptr))
    return VIDATTN_ERR_SEG_PAIR;
  int st = check_args(d_q, d_k, d_v, d_seg_q, d_seg_kv, d_out, d_lse, B, H, S_q, S_kv, D);
  if (st != VIDATTN_OK) return st;
  if (!std::isfinite(scale)) return VIDATTN_ERR_BAD_SHAPE;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const size_t qb = size_t(B) * H * S_q * D * 2, kvb = size_t(B) * H * S_kv * D * 2;
  auto h2d = [&](void* d, const void* h, size_t n) {
    return n == 0 || cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, stream) == cudaSuccess;
  };
  auto d2h = [&](void* h, const void* d, size_t n) {
    return n == 0 || cudaMemcpyAsync(h, d, n, cudaMemcpyDeviceToHost, stream) == cudaSuccess;
  };
  if (S_q == 0) return VIDATTN_OK;
  if (h_seg_q && (!h2d(d_seg_q, h_seg_q, size_t(B) * S_q * 4) ||
                  !h2d(d_seg_kv, h_seg_kv, size_t(B) * S_kv * 4)))
    return VIDATTN_ERR_CUDA;
  const size_t lseb = size_t(B) * H * S_q * 4;
  if (2 * qb + 2 * kvb < kPipelineMinBytes || H < 2) {
    if (!h2d(d_q, h_q, qb) || !h2d(d_k, h_k, kvb) || !h2d(d_v, h_v, kvb)) return VIDATTN_ERR_CUDA;
    st = vidattn_fwd(d_q, d_k, d_v, d_seg_q, d_seg_kv, d_out, d_lse, B, H, S_q, S_kv, D, scale,
                     stream_);
    if (st != VIDATTN_OK) return st;
    if (!d2h(h_out, d_out, qb) || !d2h(h_lse, d_lse, lseb)) return VIDATTN_ERR_CUDA;
    return VIDATTN_OK;
  }

  // Pipelined by chunks of heads: the copy-in of chunk c+1 and the copy-out
  // of chunk c-1 run on two copy streams while chunk c's attention runs;
  // chunks alternate between `stream` and a second compute stream, so a
  // chunk's CTAs take the SMs that the previous chunk's last wave leaves
  // idle.  Events order each chunk's copy-in, attention and copy-out.  The
  // heads are independent, so the result is the same, bit for bit.
  int dev = 0;
  st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;
  cudaStream_t cin = nullptr, cout = nullptr, comp2 = nullptr;
  if (!host_streams(dev, &cin, &cout, &comp2)) return VIDATTN_ERR_CUDA;
  const int hc = (H + kPipelineChunks - 1) / kPipelineChunks;
  // every chunk uses the whole call's key splits, so the result is the
  // device entry point's bit for bit (a chunk alone has fewer work units
  // and the heuristic could split it differently)
  const int split_flag =
      VIDATTN_SPLIT_KV(vidattn_split_count(d_seg_q, B, H, S_q, S_kv, 0));
  const size_t hq = size_t(S_q) * D * 2, hkv = size_t(S_kv) * D * 2, hl = size_t(S_q) * 4;
  auto ev = [](cudaEvent_t* e) {
    return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  };
  cudaEvent_t start = nullptr, done = nullptr;
  if (!ev(&start) || !ev(&done)) {
    if (start) cudaEventDestroy(start);
    return VIDATTN_ERR_CUDA;
  }
  bool ok = cudaEventRecord(start, stream) == cudaSuccess &&
            cudaStreamWaitEvent(cin, start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(cout, start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(comp2, start, 0) == cudaSuccess;
  int chunk = 0;
  auto* cq = static_cast<const char*>(h_q);
  auto* ck = static_cast<const char*>(h_k);
  auto* cv = static_cast<const char*>(h_v);
  for (int b = 0; ok && b < B; ++b) {
    for (int h0 = 0; ok && h0 < H; h0 += hc) {
      const int nh = (H - h0) < hc ? (H - h0) : hc;
      const size_t u = size_t(b) * H + h0;   // first (b, h) slab of the chunk
      char* dq = static_cast<char*>(d_q) + u * hq;
      char* dk = static_cast<char*>(d_k) + u * hkv;
      char* dv = static_cast<char*>(d_v) + u * hkv;
      char* dout = static_cast<char*>(d_out) + u * hq;
      float* dl = d_lse + u * S_q;
      cudaEvent_t in_done = nullptr, k_done = nullptr;
      if (!ev(&in_done) || !ev(&k_done)) {
        if (in_done) cudaEventDestroy(in_done);
        ok = false;
        break;
      }
      ok = cudaMemcpyAsync(dq, cq + u * hq, nh * hq, cudaMemcpyHostToDevice, cin) == cudaSuccess &&
           (S_kv == 0 ||
            (cudaMemcpyAsync(dk, ck + u * hkv, nh * hkv, cudaMemcpyHostToDevice, cin) ==
                 cudaSuccess &&
             cudaMemcpyAsync(dv, cv + u * hkv, nh * hkv, cudaMemcpyHostToDevice, cin) ==
                 cudaSuccess)) &&
           cudaEventRecord(in_done, cin) == cudaSuccess;
      cudaStream_t comp = (chunk++ & 1) ? comp2 : stream;
      ok = ok && cudaStreamWaitEvent(comp, in_done, 0) == cudaSuccess;
      if (ok) {
        st = vidattn_fwd_ex(dq, dk, dv, d_seg_q ? d_seg_q + size_t(b) * S_q : nullptr,
                            d_seg_kv ? d_seg_kv + size_t(b) * S_kv : nullptr, dout, dl, 1, nh,
                            S_q, S_kv, D, scale, split_flag,
                            reinterpret_cast<vidattn_stream_t>(comp));
        ok = st == VIDATTN_OK;
      }
      ok = ok && cudaEventRecord(k_done, comp) == cudaSuccess &&
           cudaStreamWaitEvent(cout, k_done, 0) == cudaSuccess &&
           cudaMemcpyAsync(static_cast<char*>(h_out) + u * hq, dout, nh * hq,
                           cudaMemcpyDeviceToHost, cout) == cudaSuccess &&
           cudaMemcpyAsync(h_lse + u * S_q, dl, nh * hl, cudaMemcpyDeviceToHost, cout) ==
               cudaSuccess;
      cudaEventDestroy(in_done);   // released once complete
      cudaEventDestroy(k_done);
    }
  }
  // `stream` waits for everything enqueued on the three side streams (a
  // stream-wait takes the event's latest record), after an error too, so
  // that the caller may free or reuse the buffers once `stream` is done
  bool joined = true;
  for (cudaStream_t side : {cin, cout, comp2})
    joined = joined && cudaEventRecord(done, side) == cudaSuccess &&
             cudaStreamWaitEvent(stream, done, 0) == cudaSuccess;
  ok = ok && joined;
  cudaEventDestroy(start);
  cudaEventDestroy(done);
  if (!ok) return st != VIDATTN_OK ? st : VIDATTN_ERR_CUDA;
  return VIDATTN_OK;
}

VIDATTN_API int vidattn_device_status(vidattn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VIDATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess)
    return VIDATTN_ERR_CUDA;
  if (v != 0) {
    int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
      return VIDATTN_ERR_CUDA;
    return VIDATTN_ERR_TIMEOUT;
  }
  return VIDATTN_OK;
}

// The forward without any allocation: like vidattn_fwd, but the segment
// summaries go to the fixed device array g_noalloc_summaries.  Its summaries
// are rewritten in full by the classifier before the attention kernel reads
// them, so nothing left there by an earlier call is ever used.  Calls on one
// device whose work overlaps on the GPU (say, on two streams at once) race on
// the array; each device has its own copy.
VIDATTN_API int vidattn_fwd_noalloc(const void* q, const void* k, const void* v,
                                    const int32_t* seg_q, const int32_t* seg_kv, void* out,
                                    float* lse, int B, int H, int S_q, int S_kv, int D,
                                    float scale, vidattn_stream_t stream_) {
  int st = check_args(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D);
  if (st != VIDATTN_OK) return st;
  if (!std::isfinite(scale)) return VIDATTN_ERR_BAD_SHAPE;
  if (S_q == 0) return VIDATTN_OK;
  const int nq = (S_q + kSegTile - 1) / kSegTile;
  const int nk = (S_kv + kSegTile - 1) / kSegTile;
  if (seg_q && size_t(B) * (size_t(nq) + size_t(nk)) > kNoAllocMaxTiles)
    return VIDATTN_ERR_SCRATCH_LIMIT;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev = 0;
  st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;
  const int4* q_sum = nullptr;
  const int4* kv_sum = nullptr;
  if (seg_q) {
    int4* buf = nullptr;
    st = noalloc_scratch(dev, &buf);
    if (st != VIDATTN_OK) return st;
    q_sum = buf;
    kv_sum = buf + size_t(B) * nq;
    dim3 grid(nq > nk ? nq : nk, B, 2);
    seg_tile_classify_kernel<<<grid, 128, 0, stream>>>(seg_q, seg_kv, buf, buf + size_t(B) * nq,
                                                       S_q, S_kv);
    if (cudaGetLastError() != cudaSuccess) return VIDATTN_ERR_CUDA;
  }
  if (D == 64)
    return launch_fwd<64>(dev, q, k, v, seg_q, seg_kv, q_sum, kv_sum, out, lse, B, H, S_q, S_kv, scale,
                          stream);
  return launch_fwd<128>(dev, q, k, v, seg_q, seg_kv, q_sum, kv_sum, out, lse, B, H, S_q, S_kv, scale,
                         stream);
}

VIDATTN_API int vidattn_rope3d(const void* q_in, const void* k_in, void* q_out, void* k_out,
                               int B, int H, int S, int D,
                               long long stride_b, long long stride_h, long long stride_s,
                               int T, int Hg, int Wg, int token_offset,
                               int d_t, int d_h, int d_w, double theta, int flags,
                               vidattn_stream_t stream_) {
  if (!q_in || !q_out || (k_in == nullptr) != (k_out == nullptr)) return VIDATTN_ERR_NULL;
  if (D != 64 && D != 128) return VIDATTN_ERR_UNSUPPORTED_D;
  if (flags & ~VIDATTN_ROPE_HALF_SPLIT) return VIDATTN_ERR_BAD_SHAPE;
  const int n_tensors = k_in ? 2 : 1;
  if (B < 1 || H < 1 || S < 1 || int64_t(n_tensors) * B * H >= (int64_t(1) << 31))
    return VIDATTN_ERR_BAD_SHAPE;
  if (T < 1 || Hg < 1 || Wg < 1 || token_offset < 0 ||
      int64_t(token_offset) + int64_t(T) * Hg * Wg > S)
    return VIDATTN_ERR_BAD_SHAPE;
  const int bands[3] = {d_t, d_h, d_w};
  for (int a = 0; a < 3; ++a)
    if (bands[a] < 0 || bands[a] % 2) return VIDATTN_ERR_BAD_SHAPE;
  if (d_t + d_h + d_w != D) return VIDATTN_ERR_BAD_SHAPE;
  if (!std::isfinite(theta) || !(theta > 0.0)) return VIDATTN_ERR_BAD_SHAPE;
  if (!aligned(q_in, 16) || !aligned(q_out, 16) || (k_in && (!aligned(k_in, 16) || !aligned(k_out, 16))))
    return VIDATTN_ERR_MISALIGNED;
  if (stride_b % 8 || stride_h % 8 || stride_s % 8) return VIDATTN_ERR_MISALIGNED;
  int dev = 0;
  int st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;

  const bool half_split = (flags & VIDATTN_ROPE_HALF_SPLIT) != 0;
  RopeParams p;
  std::memset(&p, 0, sizeof(p));
  p.in[0] = static_cast<const uint16_t*>(q_in);
  p.out[0] = static_cast<uint16_t*>(q_out);
  p.in[1] = static_cast<const uint16_t*>(k_in ? k_in : q_in);
  p.out[1] = static_cast<uint16_t*>(k_out ? k_out : q_out);
  p.sb = stride_b;
  p.sh = stride_h;
  p.ss = stride_s;
  p.n_slabs = n_tensors * B * H;
  p.S = S;
  p.div_bh = make_fastdiv(uint32_t(B) * uint32_t(H));
  p.div_h = make_fastdiv(uint32_t(H));
  p.n_video = T * Hg * Wg;
  p.hw = Hg * Wg;
  p.Hg = Hg;
  p.Wg = Wg;
  p.offset = token_offset;
  p.col_h = d_t / 2;
  p.col_w = (d_t + d_h) / 2;
  rope_tables(p, D, bands, theta, half_split);

  const int variant = (D == 128 ? 2 : 0) + (half_split ? 1 : 0);
  const int grid_max = rope_grid(dev, variant);
  if (grid_max <= 0) return VIDATTN_ERR_CUDA;
  const int n_tiles = (S + kRopeTokens - 1) / kRopeTokens;
  const int grid = n_tiles < grid_max ? n_tiles : grid_max;
  rope_variant(variant)<<<grid, kRopeThreads, 0, reinterpret_cast<cudaStream_t>(stream_)>>>(p);
  return cudaGetLastError() == cudaSuccess ? VIDATTN_OK : VIDATTN_ERR_CUDA;
}

VIDATTN_API int vidattn_selftest_timeout(int timeout_us, vidattn_stream_t stream_) {
  if (timeout_us < 1 || timeout_us > 1000000) return VIDATTN_ERR_BAD_SHAPE;
  int dev = 0;
  int st = ensure_device(&dev);
  if (st != VIDATTN_OK) return st;
  int* err = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_device_error) != cudaSuccess)
    return VIDATTN_ERR_CUDA;
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream_)>>>(
      err, 1000ull * static_cast<unsigned long long>(timeout_us));
  return cudaGetLastError() == cudaSuccess ? VIDATTN_OK : VIDATTN_ERR_CUDA;
}

VIDATTN_API void vidattn_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int prev = 0;
  cudaGetDevice(&prev);
  for (auto& kv : g_devices) {
    DeviceInfo& info = kv.second;
    if (info.copy_in || info.copy_out || info.compute2) {
      cudaSetDevice(kv.first);
      for (cudaStream_t* sp : {&info.copy_in, &info.copy_out, &info.compute2}) {
        if (*sp) {
          cudaStreamSynchronize(*sp);
          cudaStreamDestroy(*sp);
          *sp = nullptr;
        }
      }
    }
  }
  for (auto& kv : g_scratch) {
    if (kv.second.ptr) {
      cudaSetDevice(kv.first.first);
      cudaStreamSynchronize(kv.first.second);
      cudaFree(kv.second.ptr);
    }
  }
  g_scratch.clear();
  // Per-context state: the symbol addresses (device error word, the
  // no-allocation array), kernel attributes and occupancy results are looked
  // up again by the next call, so a context created after this (say, after
  // cudaDeviceReset) never sees addresses of the old one.
  g_devices.clear();
  g_noalloc_ptr.clear();
  cudaSetDevice(prev);
}

}  // extern "C"

#ifdef VIDATTN_TRACE
// Trace builds only (not part of the product ABI): where the next launches
// write their timeline stamps; NULL stops tracing.
extern "C" VIDATTN_API void vidattn_trace_set(unsigned long long* buffer) { g_trace = buffer; }
#endif
