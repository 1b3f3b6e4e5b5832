// Shared pieces of the tensor-core kernels (kernels_tc.cu, kernels_gate.cu):
// tile constants, TMA tensor-map encoding, and small device helpers.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace ttt {
namespace {

constexpr int BM = 128;          // MMA M: tokens (fb, apply) or hidden rows (grad)
constexpr int CH = 64;           // bf16 elements per 128-byte swizzle row
constexpr uint32_t KSTEP_BYTES = 32;  // 16 bf16 along K inside a K-major row

// ----------------------------------------------------------------------------
// Host: tensor maps
// ----------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor of rank 2..5 with dims[0] contiguous; box inner dim is 64
// elements (128 bytes) with the 128-byte swizzle (or 32 elements with the
// 64-byte swizzle).  Out-of-range rows read 0 and are not written.
// The outer dimensions may be listed in any stride order: a "chunk" dimension
// of stride 128 bytes placed after the row dimension makes one box land as
// consecutive [rows x 128 B] blocks, the layout the MMA descriptors expect.
bool make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
              const uint64_t* byte_strides, const uint32_t* box,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = byte_strides[i];
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Before a CTA exits, wait (bounded, ignoring the abort flag) until the last
// loads issued into each of the `nstage` ring slots have landed, so no TMA
// write can reach shared memory after the CTA is gone.  `count` is the number
// of loads issued into the ring so far (slot i % nstage, phase (i/nstage)&1).
__device__ __forceinline__ void drain_ring(uint64_t* full, int nstage, int64_t count, int* err) {
  volatile int never = 0;
  for (int64_t i = count - nstage < 0 ? 0 : count - nstage; i < count; ++i)
    mbar_wait(&full[i % nstage], (uint32_t)((i / nstage) & 1), &never, err, kErrWaitFinal);
}

// σ(x) = (1 + tanh(x/2)) / 2 with the hardware tanh approximation.
__device__ __forceinline__ float sigmoid_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

int num_sms() {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sms;
  std::lock_guard<std::mutex> lk(mu);
  if (cached[dev] == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
    cached[dev] = sms;
  }
  return cached[dev];
}

}  // namespace
}  // namespace ttt
