/*
 * vidattn: the multi-head attention forward of video diffusion transformers,
 * on NVIDIA B200 (sm_100a) — bidirectional attention masked by segment ids
 * (vidattn_fwd), with an optional causal limit (vidattn_fwd_ex) or a 3D
 * neighbourhood window (vidattn_fwd_window) — and the 3D rotary embedding of
 * q and k ahead of it (vidattn_rope3d).
 *
 * The base operation (vidax: A Unified JAX Framework for Video Generative Models on
 * Accelerator Meshes, §2 "3D RoPE, 3D VAEs, and flash attention": full
 * self-attention over multi-frame patch volumes, computed without storing the
 * query-key matrix, after FlashAttention, its reference [2]; Appendix A,
 * Table 4, group 2 "Sharding, Parallelism & Custom Kernels", row
 * "HunyuanVideo-1.5: RESOURCE_EXHAUSTED at 720p": segment ids replace a dense
 * (B,H,Sq,Sk) mask and key blocks with no valid pair are skipped):
 *
 *   for every b < B, h < H, i < S_q, with A_i = { j < S_kv : seg_q[b,i] == seg_kv[b,j] }
 *   (every j when both segment pointers are NULL):
 *     out[b,h,i,:] = sum_{j in A_i} softmax_j(scale * q[b,h,i,:] . k[b,h,j,:]) * v[b,h,j,:]
 *     lse[b,h,i]   = ln sum_{j in A_i} exp(scale * q[b,h,i,:] . k[b,h,j,:])
 *   and for A_i empty: out[b,h,i,:] = 0, lse[b,h,i] = -inf.
 *
 * Arithmetic: bf16 inputs; scores, softmax statistics and the output
 * accumulator in fp32; the softmax weights are rounded to bf16 for the
 * weights-times-values product; out is rounded once to bf16 (nearest even).
 *
 * All entry points are C ABI, thread-safe for distinct streams, and never
 * throw.  Status codes are the vidattn_status values below.
 *
 * CUDA graphs: once set up, vidattn_fwd, vidattn_fwd_ex, vidattn_fwd_window,
 * vidattn_fwd_noalloc and vidattn_rope3d enqueue kernel launches on `stream`
 * and nothing else, so they can be captured into a graph.  Set-up happens on
 * the first call on a device (kernel attributes, symbol addresses, occupancy
 * queries: host calls only) and, for the calls that use scratch (ids or a
 * window), on the first call on a stream or with a larger shape (cudaMalloc
 * after synchronising that stream, which a capture does not allow).  So make
 * one call of the largest shape on the capturing stream before capturing, or
 * use vidattn_fwd_noalloc.  vidattn_fwd_host and vidattn_device_status are
 * not for capture (events on library streams; a synchronisation).
 */
#ifndef VIDATTN_H
#define VIDATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define VIDATTN_API __attribute__((visibility("default")))
#else
#define VIDATTN_API
#endif

/* A cudaStream_t (the CUDA runtime's stream handle); NULL = legacy default stream. */
typedef struct CUstream_st* vidattn_stream_t;

typedef enum {
  VIDATTN_OK = 0,
  VIDATTN_ERR_NULL = 1,            /* a required pointer is NULL */
  VIDATTN_ERR_UNSUPPORTED_D = 2,   /* D is not 64 or 128 */
  VIDATTN_ERR_BAD_SHAPE = 3,       /* B, H, S_q or S_kv out of range */
  VIDATTN_ERR_MISALIGNED = 4,      /* q, k, v, out not 16-byte aligned; lse, seg not 4-byte */
  VIDATTN_ERR_CUDA = 5,            /* a CUDA call or launch failed */
  VIDATTN_ERR_TIMEOUT = 6,         /* a kernel wait exceeded its time limit (device_status) */
  VIDATTN_ERR_NO_DEVICE = 7,       /* the current device is not sm_100 */
  VIDATTN_ERR_SEG_PAIR = 8,        /* exactly one of seg_q, seg_kv is NULL */
  VIDATTN_ERR_SCRATCH_LIMIT = 9    /* vidattn_fwd_noalloc: shape exceeds its fixed scratch */
} vidattn_status;

/*
 * vidattn_fwd — the attention forward on device buffers.
 *
 *   q       bf16 [B,H,S_q,D]  device, contiguous (D innermost), 16-byte aligned
 *   k, v    bf16 [B,H,S_kv,D] device, contiguous, 16-byte aligned (may be NULL
 *           when S_kv == 0; q, out, lse may be NULL when S_q == 0)
 *   seg_q   int32 [B,S_q]     device, contiguous, 4-byte aligned, or NULL
 *   seg_kv  int32 [B,S_kv]    device, or NULL; NULL exactly when seg_q is NULL
 *           (both NULL = one segment: every query sees every key).
 *           Ids are arbitrary int32 values; a query sees a key iff the ids are
 *           equal (padding is simply its own id).
 *   out     bf16 [B,H,S_q,D]  device, written; 16-byte aligned
 *   lse     fp32 [B,H,S_q]    device, written; natural log of the sum of
 *           exp(scale * q.k) over the allowed keys; -inf for a row with none
 *   B, H    >= 1 and <= 65535;  S_q >= 0, S_kv >= 0;  B*H*S*D < 2^31 elements
 *           per tensor is not required (64-bit offsets), but S_q, S_kv < 2^31.
 *   D       64 or 128
 *   scale   multiplier of q.k inside the softmax (usually 1/sqrt(D)); any
 *           finite value, including 0 and negative values
 *   stream  the work is enqueued on this stream; the call does not
 *           synchronise.  Inputs must stay valid until the stream reaches it.
 *
 * Ownership: the caller owns every buffer.  When segment ids are given the
 * library keeps a small device scratch buffer per (device, stream)
 * (16 bytes per 128 tokens of seg_q and seg_kv), allocated on first use,
 * grown when a larger shape arrives (growing synchronises that stream), and
 * freed by vidattn_release().  Calls on one stream are ordered, so they never
 * share scratch in flight.
 *
 * Errors: argument errors return their status before anything is enqueued;
 * launch failures return VIDATTN_ERR_CUDA.  S_q == 0 (with the other
 * arguments valid) enqueues nothing and returns VIDATTN_OK; B or H below 1
 * is VIDATTN_ERR_BAD_SHAPE.  Kernel waits are bounded (2 s); a wait
 * that runs out sets a device error word that vidattn_device_status() reports.
 * While that word is set, the kernels of later calls on the device return at
 * once without writing their outputs, until vidattn_device_status() has
 * reported and cleared it.
 * Results are deterministic: the same inputs give bitwise the same outputs.
 */
VIDATTN_API int vidattn_fwd(const void* q, const void* k, const void* v,
                            const int32_t* seg_q, const int32_t* seg_kv,
                            void* out, float* lse,
                            int B, int H, int S_q, int S_kv, int D, float scale,
                            vidattn_stream_t stream);

/* Flags of vidattn_fwd_ex. */
#define VIDATTN_CAUSAL 1   /* key j visible to query i only if also j <= i + (S_kv - S_q) */
/* Split each 256-row query block's keys into n ranges (1 <= n <= 64), run
 * as separate work units and merged by a second kernel; 0 (the default)
 * lets the library choose (vidattn_split_count). */
#define VIDATTN_SPLIT_KV(n) (((n) & 0xFF) << 8)

/*
 * vidattn_fwd_ex — vidattn_fwd with options.  flags = 0 is exactly
 * vidattn_fwd.  flags = VIDATTN_CAUSAL adds a causal limit to the segment
 * rule: query i sees key j iff the ids match (when given) and
 * j <= i + (S_kv - S_q), the last query aligned with the last key (the
 * causal "understanding" pathway that the vidax paper, §3.1, Cosmos
 * paragraph, combines with full-attention generation in one backbone;
 * combined with segment ids this is block-diagonal causal attention).  Key
 * tiles past the limit are never loaded.  Rows that see no key give out = 0,
 * lse = -inf.  flags may also carry VIDATTN_SPLIT_KV(n) (a split count
 * above 64 is VIDATTN_ERR_BAD_SHAPE): the same result within rounding (the
 * ranges' partials are merged in fp32), for callers that know their
 * launch shape better than vidattn_split_count.  Unknown flag bits return
 * VIDATTN_ERR_BAD_SHAPE.  Other arguments, errors and ownership: as
 * vidattn_fwd; the scratch also holds a split launch's partials.
 */
VIDATTN_API int vidattn_fwd_ex(const void* q, const void* k, const void* v,
                               const int32_t* seg_q, const int32_t* seg_kv,
                               void* out, float* lse,
                               int B, int H, int S_q, int S_kv, int D, float scale, int flags,
                               vidattn_stream_t stream);

/* Flags of vidattn_fwd_window. */
#define VIDATTN_WINDOW_CLAMPED 1   /* windows shifted inside the volume at its borders */

/* Packs a token's coordinates for vidattn_fwd_window (t < 1024, h, w < 2048). */
#define VIDATTN_COORD(t, h, w) \
  ((int32_t)(((uint32_t)(t) << 22) | ((uint32_t)(h) << 11) | (uint32_t)(w)))

/*
 * vidattn_fwd_window — 3D neighbourhood (windowed) attention: the attention of
 * vidattn_fwd with each query limited to the keys in a window around its own
 * position in the video volume.  The vidax paper (Appendix A, Table 4, group 4
 * "Memory, Tiling & Execution Graphs", rows on the LTX-2.5 VAE decoder) runs
 * 3D neighbourhood attention with an 11 x 11 x 11 window and gives no
 * formula; this is the window of neighbourhood attention (Hassani et al.,
 * "Neighborhood Attention Transformer", CVPR 2023):
 *
 *   every token carries coordinates (t, h, w) in a T x Hg x Wg volume, given
 *   per token as VIDATTN_COORD(t, h, w) in coord_q [B,S_q] and coord_kv
 *   [B,S_kv] (int32, device, 4-byte aligned; any token order).  On each axis
 *   a window of odd size k (win_t, win_h, win_w) starts at c - (k-1)/2 for a
 *   query at coordinate c, or, with VIDATTN_WINDOW_CLAMPED, at that start
 *   pushed into [0, extent - k] so that queries at the borders still see k
 *   keys on that axis.  Query i sees key j iff on every axis
 *   start <= c_j <= start + k - 1; out and lse are vidattn_fwd's over those
 *   keys (a row that sees none: out 0, lse -inf).
 *
 *   win_t, win_h, win_w   odd, >= 1
 *   T, Hg, Wg             volume extents, 1..1024, 1..2048, 1..2048; every
 *                         coordinate must be below its extent (one that is
 *                         not gives unspecified values for its rows; the
 *                         coordinates are never used to address memory)
 *   S_kv                  <= 262144 (the key tiles of a CTA are listed in
 *                         shared memory)
 *   flags                 0 or VIDATTN_WINDOW_CLAMPED
 *   the rest              as vidattn_fwd.
 *
 * Key tiles (128 keys) whose coordinate box misses every window of a CTA's
 * 256 queries are never loaded; tiles inside every window skip the mask.  At
 * D = 128 the mask of a key tile whose tokens all sit at the raster position
 * of their index (token x at t = x / (Hg Wg), h = x / Wg mod Hg, w = x mod
 * Wg) with Wg >= 10 is built from the tile index alone, which is faster than
 * the general path (keys' coordinates staged in shared memory); results are
 * the same either way.  Two
 * kernels per call (tile boxes, then the attention); the tile boxes use the
 * scratch of vidattn_fwd (per device and stream).  Errors: NULL coordinates
 * return VIDATTN_ERR_NULL; bad window sizes, extents, S_kv or flag bits
 * VIDATTN_ERR_BAD_SHAPE; otherwise as vidattn_fwd.
 */
VIDATTN_API int vidattn_fwd_window(const void* q, const void* k, const void* v,
                                   const int32_t* coord_q, const int32_t* coord_kv,
                                   void* out, float* lse,
                                   int B, int H, int S_q, int S_kv, int D, float scale,
                                   int win_t, int win_h, int win_w, int T, int Hg, int Wg,
                                   int flags, vidattn_stream_t stream);

/*
 * vidattn_fwd_host — the same operation on HOST buffers, for callers whose
 * data lives in host memory.  h_* are host pointers (pinned memory gives
 * asynchronous copies; pageable memory works but the copies then block);
 * d_* are caller-owned device staging buffers of the same shapes, with the
 * alignment rules of vidattn_fwd.  Enqueued behind the work already on
 * `stream`: the ids (when given) are copied in on `stream`; then, for small
 * problems (under 64 MiB of copies, or H = 1), q, k, v are copied in, the
 * forward runs and out, lse are copied back, all on `stream`.  Larger
 * problems are pipelined over chunks of heads (up to 8 per batch entry):
 * chunk c+1's inputs are copied in and chunk c-1's outputs copied back, on
 * two copy streams the library keeps per device, while chunk c's forward
 * runs, alternately on `stream` and on a third library stream (all created
 * on first use, destroyed by vidattn_release); events order the three steps
 * of each chunk, and `stream` waits for all three streams' work (after an
 * error too, so the buffers are free once `stream` has been synchronised).
 * Either way the host outputs are valid once `stream` has been synchronised,
 * and they equal vidattn_fwd's bit for bit.  Host buffers
 * should be pinned for the copies to overlap.  h_seg_q/h_seg_kv and
 * d_seg_q/d_seg_kv follow the NULL rule of vidattn_fwd.
 */
VIDATTN_API int vidattn_fwd_host(const void* h_q, const void* h_k, const void* h_v,
                                 const int32_t* h_seg_q, const int32_t* h_seg_kv,
                                 void* h_out, float* h_lse,
                                 void* d_q, void* d_k, void* d_v,
                                 int32_t* d_seg_q, int32_t* d_seg_kv,
                                 void* d_out, float* d_lse,
                                 int B, int H, int S_q, int S_kv, int D, float scale,
                                 vidattn_stream_t stream);

/*
 * vidattn_fwd_noalloc — vidattn_fwd for callers that cannot allocate device
 * memory.  The paper has no counterpart to this entry point; it exists for
 * callers such as serving processes that hand all device memory to their own
 * pool at start-up and forbid allocation afterwards, or code running under a
 * fixed device-memory budget, for whom the on-demand scratch of vidattn_fwd
 * (a cudaMalloc on first use) is not allowed.
 *
 * Same arguments and layouts as vidattn_fwd; the caller still passes every
 * input and output.  It never splits the keys (a split launch keeps partial
 * results in scratch), so its results equal, bit for bit, those of
 * vidattn_fwd_ex with VIDATTN_SPLIT_KV(1), and those of vidattn_fwd whenever
 * vidattn_split_count() is 1.  The library allocates nothing: the segment
 * summaries use a fixed array in the library's device memory (512 KiB on every
 * GPU that loads the library, held until the process exits).  Limit, when
 * segment ids are given: B * (ceil(S_q/128) + ceil(S_kv/128)) <= 32768 (for
 * example B=1 with S_q = S_kv up to 2,097,152 tokens); larger shapes return
 * VIDATTN_ERR_SCRATCH_LIMIT before anything is enqueued.  Without segment ids
 * no scratch is used at all.
 *
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address once (cudaGetSymbolAddress); make that first call
 * before any stream capture.  Calls no cudaMalloc or cudaFree.
 * Sharing: every call on a device uses the same array, and it keeps the last
 * call's contents; each call rewrites all of the summaries it reads before
 * reading them, so nothing needs clearing.  Calls whose work overlaps on the
 * GPU (for example on two streams at once) race on the array: order them.
 */
VIDATTN_API int vidattn_fwd_noalloc(const void* q, const void* k, const void* v,
                                    const int32_t* seg_q, const int32_t* seg_kv,
                                    void* out, float* lse,
                                    int B, int H, int S_q, int S_kv, int D, float scale,
                                    vidattn_stream_t stream);

#define VIDATTN_ROPE_HALF_SPLIT 1   /* pair feature k with k + d/2 instead of 2k with 2k+1 */

/*
 * vidattn_rope3d — 3D rotary position embedding of q and k, the step right
 * before the attention in the video DiT families.  The vidax paper (§2,
 * "3D RoPE, 3D VAEs, and flash attention") rotates q and k over the time,
 * height and width axes of the video latent, keeps each family's own
 * convention (the conventions do not interchange), and prints no formula.
 * This entry point applies the rotary embedding of RoFormer (Su et al.,
 * 2021) per axis:
 *
 *   the D features of a head are cut into three contiguous bands of
 *   d_t, d_h and d_w features (in that order; each even, d_t+d_h+d_w = D; a
 *   band may be empty).  Video token n (0 <= n < T*Hg*Wg) sits at sequence
 *   index token_offset + n and has coordinates t = n / (Hg*Wg),
 *   h = (n / Wg) % Hg, w = n % Wg.  In a band of d features, pair k
 *   (0 <= k < d/2) is the features (2k, 2k+1) of the band, or (k, k + d/2)
 *   with VIDATTN_ROPE_HALF_SPLIT, and is turned by
 *   a = coord * theta^(-2k/d), coord being the token's coordinate on the
 *   band's axis:  (x, y) -> (x cos a - y sin a, x sin a + y cos a).
 *   Every other token (text, padding) is copied unchanged.
 *
 *   q_in, k_in   bf16, logical shape [B,H,S,D], element (b,h,s,f) at
 *                in + b*stride_b + h*stride_h + s*stride_s + f (features
 *                contiguous), device, 16-byte aligned; strides in elements,
 *                multiples of 8.  [B,H,S,D] contiguous is (H*S*D, S*D, D);
 *                the [B,S,H,D] output of a q/k projection is (S*H*D, D, H*D).
 *   q_out, k_out bf16 [B,H,S,D] contiguous, device, 16-byte aligned, written.
 *                Either the input itself (in place, contiguous input only)
 *                or a buffer that does not overlap it.
 *   k_in, k_out  both NULL to rotate q only.
 *   B, H >= 1; n*B*H < 2^31 for n tensors (2 with k, 1 without);
 *                D = 64 or 128.
 *   T, Hg, Wg >= 1; token_offset >= 0; token_offset + T*Hg*Wg <= S.
 *   theta        finite, > 0 (10000 in the common conventions).
 *   flags        0 or VIDATTN_ROPE_HALF_SPLIT.
 *   stream       enqueued, not synchronised.
 *
 * Arithmetic: angles in fp64 reduced to [-pi, pi], sine and cosine in fp32,
 * the rotation in fp32 from the bf16 inputs, the result rounded once to bf16
 * (nearest even).  Tokens outside the video range and coordinate 0 reproduce
 * the input bit for bit.
 *
 * Errors: argument errors return their status before anything is enqueued
 * (NULL for q_in/q_out, or for exactly one of k_in/k_out; UNSUPPORTED_D;
 * MISALIGNED for a pointer or a stride; BAD_SHAPE for the rest, unknown flag
 * bits included); VIDATTN_ERR_CUDA if the launch fails.  One kernel, no
 * allocation.
 */
VIDATTN_API int vidattn_rope3d(const void* q_in, const void* k_in, void* q_out, void* k_out,
                               int B, int H, int S, int D,
                               long long stride_b, long long stride_h, long long stride_s,
                               int T, int Hg, int Wg, int token_offset,
                               int d_t, int d_h, int d_w, double theta, int flags,
                               vidattn_stream_t stream);

/* A static, human-readable name for a status code. */
VIDATTN_API const char* vidattn_status_string(int status);

/* Synchronises `stream`, then returns VIDATTN_ERR_TIMEOUT if any kernel of
 * this library on the current device reported a timed-out wait since the last
 * call (and clears the report), VIDATTN_ERR_CUDA if synchronising failed, else
 * VIDATTN_OK. */
VIDATTN_API int vidattn_device_status(vidattn_stream_t stream);

/* Launch heuristic: the number of key splits a vidattn_fwd_ex call with
 * these arguments uses (flags as for vidattn_fwd_ex; 0 when there is nothing
 * to compute or the flags are invalid).  The attention kernel works on units
 * of (b, h, 256 query rows), longest first under the causal limit: one CTA
 * per unit, or, at D = 128 with more units than SMs and at most 64 key tiles
 * (short units, whose epilogues then overlap the next unit's loads),
 * persistent with one CTA per SM looping over units.  When a call
 * has fewer than 74 such units (half of the B200's 148 SMs) the library
 * splits every unit's key tiles into ceil(148 / units) ranges (at most 16,
 * at least 8 key tiles each: shorter ranges cost more in the merge than they
 * gain), unless VIDATTN_SPLIT_KV asks for a number;
 * each range is a unit of its own, and a second kernel merges the ranges'
 * partial results (O / l and log-sum-exp per row, fp32, in the library's
 * scratch: 4 * (D + 1) bytes per row, head and split).  With segment ids and
 * more than 2048 key tiles nothing is split.  Pure host logic; no CUDA call. */
VIDATTN_API int vidattn_split_count(const int32_t* seg_q, int B, int H, int S_q, int S_kv,
                                    int flags);

/* The launch a vidattn_fwd_ex call with these arguments would make on the
 * current device (vidattn_split_count's splits, the persistent-grid choice
 * above, and the attention kernel's grid): *grid_ctas CTAs, *key_splits
 * key ranges per query block, *persistent 1 when each CTA loops over units.
 * Queries the device's SM count (a CUDA call; no launch, no allocation).
 * Returns VIDATTN_OK, or NULL / UNSUPPORTED_D / BAD_SHAPE (also for S_q < 1)
 * / NO_DEVICE / CUDA errors, leaving the outputs unset. */
VIDATTN_API int vidattn_launch_plan(const int32_t* seg_q, int B, int H, int S_q, int S_kv,
                                    int D, int flags, int* grid_ctas, int* key_splits,
                                    int* persistent);

/* Number of kernels one vidattn_fwd_ex call with these arguments launches
 * (0 when there is nothing to compute): the attention kernel, plus the tile
 * classifier with segment ids, plus the merge of a split launch.
 * Pure host logic; no CUDA call. */
VIDATTN_API int vidattn_kernels_per_call(const int32_t* seg_q, const int32_t* seg_kv,
                                         int B, int H, int S_q, int S_kv, int D, int flags);

/* Failure-detection self-test: enqueues a one-warp kernel that waits, with the
 * attention kernel's own bounded wait, on an mbarrier that nothing arrives on.
 * After timeout_us microseconds (1 .. 1e6) the wait gives up, the kernel
 * records the timeout in the device error word and returns, so a following
 * vidattn_device_status() reports VIDATTN_ERR_TIMEOUT.  Nothing faults or
 * hangs; the CUDA context stays usable. */
VIDATTN_API int vidattn_selftest_timeout(int timeout_us, vidattn_stream_t stream);

/* Frees the library's scratch buffers and destroys its internal streams (the
 * copy and second compute streams of vidattn_fwd_host) on every device, after
 * synchronising the streams concerned, and forgets what it learnt about each
 * device's CUDA context (symbol addresses, kernel attributes).  Call it while
 * no other thread is inside a vidattn call; later calls set up and allocate
 * again on demand.  Call it before cudaDeviceReset (or anything else that
 * destroys a device's primary context) if the library is used again
 * afterwards: without it the library would keep using addresses of the
 * destroyed context. */
VIDATTN_API void vidattn_release(void);

/* Library version and the GPU architecture it was compiled for. */
VIDATTN_API const char* vidattn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VIDATTN_H */
