// Unit probes of the attention kernel's building blocks, for the GPU tests
// only (built into libvidattn_probes.so, not part of the product ABI).
//
// probe_qk_pv runs, in one CTA, exactly the tensor-core steps of the forward
// kernel on one tile: TMA loads of a Q, a K and a V tile (128 rows, 128-byte
// swizzle), S = Q K^T through issue_qk (tcgen05.mma, A and B from shared
// memory), then P (given, bf16) written to tensor memory with the same packing
// the softmax uses, and O = P V through issue_pv (A from tensor memory, V as an
// MN-major shared-memory operand).  S and O are copied out in fp32 so a test
// can compare them with plain matrix products.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "fwd_kernel.cuh"

namespace vidattn {
namespace {

template <int D>
__global__ void __launch_bounds__(128, 1)
    probe_qk_pv_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const uint16_t* __restrict__ P,
                       float* __restrict__ S_out, float* __restrict__ O_out, int* status) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t sbase = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_base);
  const uint32_t sQ = sbase, sK = sbase + C::kTileBytes, sV = sbase + 2 * C::kTileBytes;
  const uint32_t bar_load = sbase + 3 * C::kTileBytes;
  const uint32_t bar_mma = bar_load + 8;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 3 * C::kTileBytes + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 3 * C::kTileBytes + 20);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(slot);

  // Warp 0 issues, converged: issue_qk / issue_pv elect one lane per MMA,
  // and the commits elect the same lane (a commit tracks its own thread's MMAs).
  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_load, 3 * C::kTileBytes);
      for (int s = 0; s < C::kSub; ++s) {
        tma_load_3d(sQ + s * C::kSubBytes, &tm_q, bar_load, s * 64, 0, 0);
        tma_load_3d(sK + s * C::kSubBytes, &tm_k, bar_load, s * 64, 0, 0);
        tma_load_3d(sV + s * C::kSubBytes, &tm_v, bar_load, s * 64, 0, 0);
      }
    }
    __syncwarp();
    ok = warp_wait_phase(bar_load, 0, abort_flag, status, 100000000ull);
    if (ok) {
      tc_fence_after();
      issue_qk<D>(tmem + 0, sQ, sK);
      mma_commit_elect(bar_mma);
    }
  }
  ok = __syncthreads_and(ok);
  ok = ok && wait_phase(bar_mma, 0, abort_flag, status, 100000000ull);
  ok = __all_sync(0xffffffffu, ok);
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int r = warp * 32 + lane;
  if (ok) {
    tc_fence_after();
    for (int k = 0; k < 4; ++k) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + 32 * k, v);
      tmem_ld_wait();
      reg_fence(v);
      for (int x = 0; x < 32; ++x) S_out[r * 128 + 32 * k + x] = __uint_as_float(v[x]);
    }
    // P row r -> tensor memory columns [256, 320), two bf16 per column
    uint32_t pk[2][32];
    for (int x = 0; x < 64; ++x) {
      const uint32_t lo = P[r * 128 + 2 * x], hi = P[r * 128 + 2 * x + 1];
      pk[x >> 5][x & 31] = lo | (hi << 16);
    }
    tmem_st32(tmem + lane_off + 256, pk[0]);
    tmem_st32(tmem + lane_off + 256 + 32, pk[1]);
    tmem_st_wait();
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (ok && warp == 0) {
    tc_fence_after();
    issue_pv<D>(tmem + 384, tmem + 256, sV, false);
    mma_commit_elect(bar_mma);
  }
  ok = ok && wait_phase(bar_mma, 1, abort_flag, status, 100000000ull);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    for (int k = 0; k < D / 32; ++k) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + 384 + 32 * k, v);
      tmem_ld_wait();
      reg_fence(v);
      for (int x = 0; x < 32; ++x) O_out[r * D + 32 * k + x] = __uint_as_float(v[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// y[i] = exp2_poly2 of x[i] (pairs), the FMA-pipe exponential of the softmax.
__global__ void probe_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
}

bool encode(CUtensorMap* m, const void* ptr, int D) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), 128, 1};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(D) * 2 * 128};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace vidattn

using namespace vidattn;

// q, k, v: bf16 [128, D] device; P: bf16 [128,128] device; S_out: fp32
// [128,128]; O_out: fp32 [128, D]; status: device int (bit 1 = a wait timed
// out).  Returns 0 on a successful launch.
extern "C" __attribute__((visibility("default"))) int probe_qk_pv(
    const void* q, const void* k, const void* v, const void* P, float* S_out, float* O_out,
    int* status, int D, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (D != 64 && D != 128) return 2;
  if (!encode(&tq, q, D) || !encode(&tk, k, D) || !encode(&tv, v, D)) return 3;
  const int smem = 3 * 128 * D * 2 + 64 + 1024;
  if (D == 64) {
    cudaFuncSetAttribute(probe_qk_pv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    probe_qk_pv_kernel<64><<<1, 128, smem, stream>>>(tq, tk, tv, static_cast<const uint16_t*>(P),
                                                      S_out, O_out, status);
  } else {
    cudaFuncSetAttribute(probe_qk_pv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         smem);
    probe_qk_pv_kernel<128><<<1, 128, smem, stream>>>(tq, tk, tv, static_cast<const uint16_t*>(P),
                                                       S_out, O_out, status);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

// x, y: n fp32 device values (n even).
extern "C" __attribute__((visibility("default"))) int probe_exp2_poly(const float* x, float* y,
                                                                       int n,
                                                                       cudaStream_t stream) {
  if (n <= 0 || (n & 1)) return 2;
  const int pairs = n / 2;
  probe_exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}
