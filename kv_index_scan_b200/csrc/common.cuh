// common.cuh -- shared helpers of libkvscan (host error plumbing, small device
// utilities). Every kernel of the library is written for sm_100a.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>

#include "kvscan.h"

namespace kvs {

// ----------------------------------------------------------------------------- host errors

// Records a printf-style message as this thread's last error and returns st.
kvs_status fail(kvs_status st, const char* fmt, ...);
// KVS_OK after clearing this thread's message.
kvs_status ok();
// Maps the last launch error of this thread to KVS_ECUDA (with its text).
kvs_status check_launch(const char* what);

#define KVS_REQUIRE(cond, st, ...)          \
  do {                                      \
    if (!(cond)) return ::kvs::fail(st, __VA_ARGS__); \
  } while (0)

// ----------------------------------------------------------------------------- launch chaining
// The kernels of a decode step are launched with programmatic stream
// serialization: a kernel may be launched while its predecessor in the stream
// still runs (once every block of the predecessor has called pdl_trigger), so
// that its launch and ramp overlap the predecessor's tail. Every such kernel
// calls pdl_wait before its first global memory access: it returns once the
// predecessor has completed and its writes are visible (at once when the
// kernel was not launched that way).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" :::); }

template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves consecutive 256-byte aligned regions out of a caller workspace.
struct WsCarver {
  char* base;
  size_t used = 0;
  explicit WsCarver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    used = align_up(used, 256);
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used += count * sizeof(T);
    return p;
  }
};

// Number of SMs of the current device (cached per device).
int sm_count();

// ----------------------------------------------------------------------------- device helpers

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Monotone map f32 -> u32: a > b (as floats, no NaN) <=> key(a) > key(b), and
// a == b <=> key(a) == key(b) (-0 is first turned into +0).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t b = __float_as_uint(__fadd_rn(f, 0.0f));
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

__device__ __forceinline__ void set_status(int32_t* dev_status, int32_t st) {
  if (dev_status) atomicCAS(dev_status, 0, st);
}

constexpr int kD = 128;  // head dim of every kernel here

}  // namespace kvs
