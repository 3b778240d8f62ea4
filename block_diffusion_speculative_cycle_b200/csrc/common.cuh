// Shared device helpers for the DFlash draft-cycle kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace dfl {

// ---------------------------------------------------------------- status bits
// Kernels record problems here and skip the offending element; they never trap.
enum : int {
  ST_BAD_TOKEN = 1,     // a token id outside [0, V)
  ST_BAD_PAGE = 2,      // a page id outside [0, num_pages) or a page slot beyond max_pages
  ST_TIMEOUT = 4,       // a bounded wait gave up
  ST_BAD_CTX = 8,       // a context length outside [0, max_ctx]
};

__device__ __forceinline__ void flag_error(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------- element conversion
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------- argmax keys
// A (value, index) pair packed so that the unsigned 64-bit maximum is the
// largest value and, among equal values, the lowest index. NaN ranks below
// every number (-inf included) and -0.0 equals +0.0. atomicMax on these keys is
// order-independent, hence deterministic.
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  unsigned int u;
  if (v != v) {
    u = 0u;
  } else {
    if (v == 0.0f) v = 0.0f;
    unsigned int b = __float_as_uint(v);
    u = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  return ((unsigned long long)u << 32) | (unsigned long long)(~(unsigned int)idx);
}
__device__ __forceinline__ int argmax_key_index(unsigned long long key) {
  return (int)(~(unsigned int)(key & 0xffffffffull));
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  unsigned int lo = (unsigned int)v, hi = (unsigned int)(v >> 32);
  lo = __shfl_xor_sync(0xffffffffu, lo, m);
  hi = __shfl_xor_sync(0xffffffffu, hi, m);
  return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    unsigned long long o = shfl_xor_u64(v, m);
    v = o > v ? o : v;
  }
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// ---------------------------------------------------------------- time
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Every spin in these kernels gives up after this long and flags ST_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------- RoPE
// Rotate-half RoPE factors for a pair with inverse frequency inv_freq (double,
// theta^(-2i/d)) at integer position pos. The angle pos*inv_freq is formed and
// reduced to [-pi, pi] in double (one multiply, one rounding, one fma), so that
// positions up to 2^24 keep full fp32 accuracy; cos/sin are then taken in fp32.
// The double arithmetic is slow on this part: the GEMM epilogues read (cos, sin)
// from a per-row table filled once per call (RopeFill below) instead.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double two_pi = 6.283185307179586;
  const double a = (double)pos * inv_freq;
  const double k = rint(a * (1.0 / two_pi));
  const float r = (float)fma(-k, two_pi, a);
  sincosf(r, s, c);
}

// The per-row RoPE table of one call: out[m * half + i] = (cos, sin) of the angle
// of row m's position, pos_base[m / rows_per_req] + m % rows_per_req, at
// inv_freq[i], for rows m < rows (out null: nothing to fill).
struct RopeFill {
  const int* pos_base;
  int rows_per_req;
  int rows;
  int half;
  const double* inv_freq;
  float2* out;
};

__device__ __forceinline__ void rope_fill_entry(const RopeFill& f, int e) {
  const int m = e / f.half, i = e % f.half;
  const int pos = __ldg(f.pos_base + m / f.rows_per_req) + m % f.rows_per_req;
  float c, s;
  rope_cos_sin(pos, __ldg(f.inv_freq + i), &c, &s);
  f.out[e] = make_float2(c, s);
}
// entries first, first + stride, ... of the whole table
__device__ __forceinline__ void rope_fill_range(const RopeFill& f, int first, int stride) {
  if (!f.out) return;
  const int n = f.rows * f.half;
  for (int e = first; e < n; e += stride) rope_fill_entry(f, e);
}

// silu(g) = g * sigmoid(g), with the fast exponential and divide intrinsics
// (relative error ~1e-6, well below the bf16 hi/lo output's resolution).
// For g < -88, __expf(-g) is +inf and the quotient is -0.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// ---------------------------------------------------------------- programmatic dependent launch
// With PDL a kernel may start while its predecessor in the stream is still
// running; it must not touch the predecessor's data before grid_dep_wait().
// Without PDL both are no-ops.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with the programmatic-stream-serialization attribute when pdl is set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace dfl
