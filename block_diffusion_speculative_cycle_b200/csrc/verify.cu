// Greedy verify of a drafted block against the target's block logits.
//
// Grid (chunk, row j, request b): each CTA streams one chunk of one logits row
// with 16-byte loads, reduces a packed (value, index) key and folds it into
// keys[b, j] with atomicMax (order-independent, so bit-reproducible). The last
// CTA of a request (atomic ticket) walks the B rows: a = leading matches of
// draft[i-1] against argmax row i-1, next = argmax row a; it then zeroes the
// request's keys and ticket so the workspace is ready for the next call.
#include <cstdio>
#include "trace.h"
#include <cstdlib>
#include <mutex>

#include "../../include/dflash.h"
#include "common.cuh"

namespace dfl {

constexpr int kVerifyThreads = 256;
constexpr int kVerifyChunk = 8192;   // logits per CTA

template <typename T>
__device__ __forceinline__ unsigned long long chunk_best(const T* row, int v0, int v1);

template <>
__device__ __forceinline__ unsigned long long chunk_best<__nv_bfloat16>(const __nv_bfloat16* row, int v0, int v1) {
  unsigned long long best = 0ull;
  // 8 bf16 per 16-byte load when the chunk start is 16-byte aligned
  const bool vec = ((reinterpret_cast<uintptr_t>(row + v0) & 15) == 0);
  int v = v0;
  if (vec) {
    const int nvec = (v1 - v0) / 8;
    const uint4* p = reinterpret_cast<const uint4*>(row + v0);
#pragma unroll 4
    for (int e = threadIdx.x; e < nvec; e += blockDim.x) {
      const uint4 u = __ldcs(p + e);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xffff0000u);
        const int idx = v0 + e * 8 + 2 * k;
        unsigned long long a = argmax_key(lo, idx), b = argmax_key(hi, idx + 1);
        a = a > b ? a : b;
        best = a > best ? a : best;
      }
    }
    v = v0 + nvec * 8;
  }
  for (int e = v + threadIdx.x; e < v1; e += blockDim.x) {
    const unsigned long long a = argmax_key(__bfloat162float(row[e]), e);
    best = a > best ? a : best;
  }
  return best;
}

template <>
__device__ __forceinline__ unsigned long long chunk_best<float>(const float* row, int v0, int v1) {
  unsigned long long best = 0ull;
  const bool vec = ((reinterpret_cast<uintptr_t>(row + v0) & 15) == 0);
  int v = v0;
  if (vec) {
    const int nvec = (v1 - v0) / 4;
    const float4* p = reinterpret_cast<const float4*>(row + v0);
#pragma unroll 4
    for (int e = threadIdx.x; e < nvec; e += blockDim.x) {
      const float4 f = __ldcs(p + e);
      const float w[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const unsigned long long a = argmax_key(w[k], v0 + e * 4 + k);
        best = a > best ? a : best;
      }
    }
    v = v0 + nvec * 4;
  }
  for (int e = v + threadIdx.x; e < v1; e += blockDim.x) {
    const unsigned long long a = argmax_key(row[e], e);
    best = a > best ? a : best;
  }
  return best;
}

template <typename T>
__global__ void __launch_bounds__(kVerifyThreads) verify_kernel(const T* logits, const int* draft, int B, int V,
                                                                 unsigned long long* keys, int* tickets,
                                                                 int* accepted, int* next_token) {
  __shared__ unsigned long long red[kVerifyThreads / 32];
  __shared__ int s_last;
  grid_dep_wait();
  grid_dep_launch();
  const int c = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const T* row = logits + ((size_t)b * B + j) * V;
  const int v0 = c * kVerifyChunk, v1 = min(V, v0 + kVerifyChunk);
  unsigned long long best = warp_max_u64(chunk_best<T>(row, v0, v1));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kVerifyThreads / 32; ++w) best = red[w] > best ? red[w] : best;
    atomicMax(keys + (size_t)b * B + j, best);
    __threadfence();
    const int total = (int)gridDim.x * B;
    s_last = atomicAdd(tickets + b, 1) == total - 1;
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  // the request's last CTA: warp 0 tests 32 drafts per round trip. Lane i of a
  // round compares draft i with the argmax of row i; a = the leading matches.
  __threadfence();
  unsigned long long* kb = keys + (size_t)b * B;
  const int* dr = draft + (size_t)b * (B - 1);
  int a = 0;
  for (int i0 = 0; i0 < B - 1; i0 += 32) {
    const int i = i0 + lane, nv = min(32, B - 1 - i0);
    const bool match = i < B - 1 && __ldg(dr + i) == argmax_key_index(__ldcg(kb + i));
    const unsigned miss = ~__ballot_sync(0xffffffffu, match);
    const int lead = miss ? __ffs((int)miss) - 1 : 32;   // lanes >= nv count as misses
    a += lead;
    if (lead < nv) break;
  }
  if (lane == 0) {
    accepted[b] = a;
    next_token[b] = argmax_key_index(__ldcg(kb + a));
  }
  __syncwarp();
  // leave the request's keys and ticket zeroed for the next call
  for (int r = lane; r < B; r += 32) kb[r] = 0ull;
  if (lane == 0) tickets[b] = 0;
}

// Programmatic dependent launch for verify (on unless DFLASH_PDL=0).
static bool verify_pdl() {
  static const bool on = [] {
    const char* e = std::getenv("DFLASH_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <typename T>
static cudaError_t launch_verify(const T* logits, const int* draft, int bs, int B, int V, unsigned long long* keys,
                                 int* tickets, int* accepted, int* next_token, cudaStream_t st) {
  const dim3 grid((unsigned)((V + kVerifyChunk - 1) / kVerifyChunk), (unsigned)B, (unsigned)bs);
  return launch_kernel(verify_kernel<T>, grid, dim3(kVerifyThreads), 0, st, verify_pdl(), logits, draft, B, V, keys,
                       tickets, accepted, next_token);
}

}  // namespace dfl

extern "C" size_t dflash_verify_workspace_size(int bs, int B) {
  if (bs <= 0 || B <= 0) return 0;
  const size_t keys = (size_t)bs * B * sizeof(unsigned long long);
  return keys + (((size_t)bs * sizeof(int) + 255) / 256) * 256;
}

extern "C" dflash_status dflash_verify(const void* d_logits, dflash_dtype logits_dtype, const int* d_draft, int bs,
                                       int B, int V, int* d_accepted, int* d_next_token, void* d_workspace,
                                       size_t workspace_bytes, void* stream) {
  dfl::TraceRange trace_("dflash_verify");
  if (bs <= 0 || B <= 0 || V <= 0 || !d_logits || !d_accepted || !d_next_token || !d_workspace) return DFLASH_ERR_ARG;
  if (B > 1 && !d_draft) return DFLASH_ERR_ARG;
  if (logits_dtype != DFLASH_F32 && logits_dtype != DFLASH_BF16) return DFLASH_ERR_ARG;
  if (workspace_bytes < dflash_verify_workspace_size(bs, B)) return DFLASH_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(d_workspace) & 7) != 0) return DFLASH_ERR_ARG;
  if (bs > 65535 || B > 65535) return DFLASH_ERR_UNSUPPORTED;
  auto* keys = reinterpret_cast<unsigned long long*>(d_workspace);
  auto* tickets = reinterpret_cast<int*>(reinterpret_cast<char*>(d_workspace) + (size_t)bs * B * 8);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e =
      logits_dtype == DFLASH_BF16
          ? dfl::launch_verify((const __nv_bfloat16*)d_logits, d_draft, bs, B, V, keys, tickets, d_accepted,
                               d_next_token, st)
          : dfl::launch_verify((const float*)d_logits, d_draft, bs, B, V, keys, tickets, d_accepted, d_next_token, st);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}

// ---------------------------------------------------------------- no-allocation variant
// Scratch of dflash_verify_noalloc: keys at offset 0, tickets after the keys.
// A host-side mention of this name is only a stand-in symbol, not a device
// address; host code passes the address from cudaGetSymbolAddress instead.
static __device__ __align__(256) unsigned char g_verify_scratch[DFLASH_VERIFY_NOALLOC_MAX_ROWS * 8 +
                                                                 DFLASH_VERIFY_NOALLOC_MAX_BATCH * 4];

namespace {
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_verify_scratch on the current device, looked up once per device.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_verify_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}
}  // namespace

extern "C" dflash_status dflash_verify_noalloc(const void* d_logits, dflash_dtype logits_dtype, const int* d_draft,
                                               int bs, int B, int V, int* d_accepted, int* d_next_token,
                                               void* stream) {
  dfl::TraceRange trace_("dflash_verify_noalloc");
  if (bs <= 0 || B <= 0 || V <= 0 || !d_logits || !d_accepted || !d_next_token) return DFLASH_ERR_ARG;
  if (B > 1 && !d_draft) return DFLASH_ERR_ARG;
  if (logits_dtype != DFLASH_F32 && logits_dtype != DFLASH_BF16) return DFLASH_ERR_ARG;
  if (bs > DFLASH_VERIFY_NOALLOC_MAX_BATCH || (long long)bs * B > DFLASH_VERIFY_NOALLOC_MAX_ROWS) {
    std::fprintf(stderr,
                 "dflash_verify_noalloc: bs=%d, B=%d exceed the fixed scratch (bs <= %d, bs*B <= %d); "
                 "use dflash_verify with a caller-provided workspace\n",
                 bs, B, DFLASH_VERIFY_NOALLOC_MAX_BATCH, DFLASH_VERIFY_NOALLOC_MAX_ROWS);
    return DFLASH_ERR_ARG;
  }
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return DFLASH_ERR_CUDA;
  auto* keys = reinterpret_cast<unsigned long long*>(scratch);
  auto* tickets = reinterpret_cast<int*>(reinterpret_cast<char*>(scratch) + DFLASH_VERIFY_NOALLOC_MAX_ROWS * 8);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(keys, 0, (size_t)bs * B * 8, st) != cudaSuccess) return DFLASH_ERR_CUDA;
  if (cudaMemsetAsync(tickets, 0, (size_t)bs * 4, st) != cudaSuccess) return DFLASH_ERR_CUDA;
  const dim3 grid((unsigned)((V + dfl::kVerifyChunk - 1) / dfl::kVerifyChunk), (unsigned)B, (unsigned)bs);
  if (logits_dtype == DFLASH_BF16)
    dfl::verify_kernel<__nv_bfloat16><<<grid, dfl::kVerifyThreads, 0, st>>>(
        (const __nv_bfloat16*)d_logits, d_draft, B, V, keys, tickets, d_accepted, d_next_token);
  else
    dfl::verify_kernel<float><<<grid, dfl::kVerifyThreads, 0, st>>>((const float*)d_logits, d_draft, B, V, keys,
                                                                    tickets, d_accepted, d_next_token);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
