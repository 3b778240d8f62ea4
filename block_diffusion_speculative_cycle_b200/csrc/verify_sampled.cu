// Sampled (temperature > 0) verification of a drafted block.
//
// The rule ("DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩" §1: drafts the
// target agrees with are kept; from the first one it does not, the target's own
// distribution decides, so the output follows target-only sampling; the
// standard speculative-sampling scheme the page names), position by position:
// with p_j = softmax(Z_j / T) the target's distribution at block row j and
// q_i = softmax(Y_{i-1} / T) the distribution draft d_i was drawn from,
//   d_i is accepted while u_accept[i-1] * q_i(d_i) < p_{i-1}(d_i)   (i = 1 .. B-1);
//   at the first rejection i = a+1 the next token is drawn from the residual
//   max(0, p_a - q_{a+1}), normalised (p_a itself if that is zero everywhere);
//   when all B-1 drafts pass, it is drawn from p_{B-1};
// a draw takes the smallest index v whose running sum (index order) exceeds
// u_final * total.
//
// Two kernels, no inter-CTA waits (a ticket elects the last CTA of a request):
//   sv_stats  grid (chunk, row, request): per vocabulary chunk of every target
//             row and draft row, the chunk's max of x/T and sum of exp(x/T - max);
//   sv_decide grid (chunk, request): every CTA merges the chunk statistics into
//             each row's log-sum-exp in chunk order, decides a (all CTAs alike),
//             and sums its chunk of the distribution to draw from; the last CTA
//             of the request finds the chunk, then the entry, where the running
//             sum crosses u_final * total, writes (a, next) and resets its ticket.
// All sums are taken in fixed orders, so the results are reproducible run to run.
#include <cmath>
#include <cstdio>

#include "../../include/dflash.h"
#include "common.cuh"
#include "trace.h"

namespace dfl {

namespace {

constexpr int kSvThreads = 256;
constexpr int kSvChunk = 8192;   // vocabulary entries per CTA
constexpr int kSvSeg = kSvChunk / kSvThreads;   // contiguous entries per thread (32)

template <typename T> __device__ __forceinline__ float ld(const T* p) { return to_f32(__ldg(p)); }
template <> __device__ __forceinline__ float ld<float>(const float* p) { return __ldg(p); }

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kSvThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}
// Sum over the block in a fixed order: warps in index order, lanes by butterfly.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < kSvThreads / 32; ++i) r += red[i];
  return r;
}

}  // namespace

// stats[((b * (2B-1) + r) * nch + c) * 2 + {0, 1}] = (max x/T, sum exp(x/T - max)) over chunk c of row r:
// rows r < B are target rows Z[b, r], rows r >= B are draft rows Y[b, r - B].
template <typename TZ>
__global__ void __launch_bounds__(kSvThreads) sv_stats_kernel(const TZ* Z, const float* Y, int B, int V, float inv_t,
                                                              float* stats) {
  __shared__ float red[kSvThreads / 32];
  const int c = blockIdx.x, r = blockIdx.y, b = blockIdx.z, nch = gridDim.x;
  const int v0 = c * kSvChunk, v1 = min(V, v0 + kSvChunk);
  float mx = -INFINITY;
  if (r < B) {
    const TZ* row = Z + ((size_t)b * B + r) * V;
    for (int v = v0 + threadIdx.x; v < v1; v += kSvThreads) mx = fmaxf(mx, ld(row + v) * inv_t);
  } else {
    const float* row = Y + ((size_t)b * (B - 1) + (r - B)) * V;
    for (int v = v0 + threadIdx.x; v < v1; v += kSvThreads) mx = fmaxf(mx, ld(row + v) * inv_t);
  }
  mx = block_max(mx, red);
  float sum = 0.f;
  if (mx != -INFINITY) {
    if (r < B) {
      const TZ* row = Z + ((size_t)b * B + r) * V;
      for (int v = v0 + threadIdx.x; v < v1; v += kSvThreads) sum += __expf(ld(row + v) * inv_t - mx);
    } else {
      const float* row = Y + ((size_t)b * (B - 1) + (r - B)) * V;
      for (int v = v0 + threadIdx.x; v < v1; v += kSvThreads) sum += __expf(ld(row + v) * inv_t - mx);
    }
  }
  sum = block_sum(sum, red);
  if (threadIdx.x == 0) {
    float* o = stats + (((size_t)b * (2 * B - 1) + r) * nch + c) * 2;
    o[0] = mx;
    o[1] = sum;
  }
}

namespace {

// log-sum-exp of row r from its chunk statistics, merged in chunk order.
__device__ __forceinline__ float row_lse(const float* stats, int b, int B, int r, int nch) {
  const float* s = stats + ((size_t)b * (2 * B - 1) + r) * nch * 2;
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(s + 2 * c));
  float L = 0.f;
  for (int c = 0; c < nch; ++c) {
    const float m = __ldcg(s + 2 * c);
    if (m != -INFINITY) L += __ldcg(s + 2 * c + 1) * __expf(m - M);
  }
  return M + __logf(L);
}

}  // namespace

// The value the draw is taken over at vocabulary entry v: the residual
// max(0, p_a - q_{a+1}) after a rejection (mode 0), or p_a itself (mode 1: all
// drafts accepted, or an all-zero residual).
template <typename TZ>
__device__ __forceinline__ float draw_weight(const TZ* zrow, const float* yrow, float inv_t, float lse_z, float lse_y,
                                             int v, int mode) {
  const float pz = __expf(ld(zrow + v) * inv_t - lse_z);
  if (mode) return pz;
  return fmaxf(0.f, pz - __expf(ld(yrow + v) * inv_t - lse_y));
}

template <typename TZ>
__global__ void __launch_bounds__(kSvThreads) sv_decide_kernel(const TZ* Z, const float* Y, const int* draft, int B,
                                                               int V, float inv_t, const float* u_accept,
                                                               const float* u_final, const float* stats,
                                                               float* chunk_sum, int* tickets, int* accepted,
                                                               int* next_token) {
  __shared__ float red[kSvThreads / 32];
  __shared__ int s_a, s_mode, s_last;
  __shared__ float s_lz, s_ly;
  grid_dep_wait();
  grid_dep_launch();
  const int c = blockIdx.x, b = blockIdx.y, nch = gridDim.x;
  if (threadIdx.x == 0) {
    // the accepted prefix: every CTA of the request decides it the same way
    int a = 0;
    while (a < B - 1) {
      const int d = draft[(size_t)b * (B - 1) + a];
      bool ok = d >= 0 && d < V;
      if (ok) {
        const float pd = __expf(ld(Z + ((size_t)b * B + a) * V + d) * inv_t - row_lse(stats, b, B, a, nch));
        const float qd = __expf(ld(Y + ((size_t)b * (B - 1) + a) * V + d) * inv_t - row_lse(stats, b, B, B + a, nch));
        ok = __ldg(u_accept + (size_t)b * (B - 1) + a) * qd < pd;
      }
      if (!ok) break;
      ++a;
    }
    s_a = a;
    s_mode = a == B - 1 ? 1 : 0;
    s_lz = row_lse(stats, b, B, a, nch);
    s_ly = a < B - 1 ? row_lse(stats, b, B, B + a, nch) : 0.f;
  }
  __syncthreads();
  const int a = s_a;
  const TZ* zrow = Z + ((size_t)b * B + a) * V;
  const float* yrow = a < B - 1 ? Y + ((size_t)b * (B - 1) + a) * V : nullptr;
  const float lz = s_lz, ly = s_ly;
  // this chunk's total, thread segments of kSvSeg contiguous entries summed in order
  const int v0 = c * kSvChunk;
  auto seg_sum = [&](int mode) {
    float t = 0.f;
    const int s0 = v0 + threadIdx.x * kSvSeg, s1 = min(V, s0 + kSvSeg);
    for (int v = s0; v < s1; ++v) t += draw_weight(zrow, yrow, inv_t, lz, ly, v, mode);
    return t;
  };
  const float tot = block_sum(seg_sum(s_mode), red);
  if (threadIdx.x == 0) {
    chunk_sum[(size_t)b * nch + c] = tot;
    __threadfence();
    s_last = atomicAdd(tickets + b, 1) == nch - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last CTA of the request: the chunk, then the entry, where the running sum crosses the target
  int mode = s_mode;
  float total = 0.f;
  for (int k = 0; k < nch; ++k) total += __ldcg(chunk_sum + (size_t)b * nch + k);
  if (!(total > 0.f) && mode == 0) mode = 1;   // residual zero everywhere: draw from p_a
  __shared__ int s_chunk;
  __shared__ float s_before;
  if (threadIdx.x == 0) {
    const float target = __ldg(u_final + b) * (mode == s_mode ? total : 1.f);
    int ck = nch - 1;
    float run = 0.f;
    if (mode == s_mode) {
      for (int k = 0; k < nch; ++k) {
        const float cs = __ldcg(chunk_sum + (size_t)b * nch + k);
        if (run + cs > target) {
          ck = k;
          break;
        }
        run += cs;
      }
    } else {
      ck = -1;   // fallback: scan the whole row below
    }
    s_chunk = ck;
    s_before = run;
  }
  __syncthreads();
  int next = -1;
  if (s_chunk >= 0) {
    // segment sums of the chosen chunk, in thread order, then the entry
    const int cv0 = s_chunk * kSvChunk;
    float t = 0.f;
    const int s0 = cv0 + threadIdx.x * kSvSeg, s1 = min(V, s0 + kSvSeg);
    for (int v = s0; v < s1; ++v) t += draw_weight(zrow, yrow, inv_t, lz, ly, v, mode);
    __shared__ float segs[kSvThreads];
    segs[threadIdx.x] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
      const float target = __ldg(u_final + b) * total;
      float run = s_before;
      int last_pos = -1;
      for (int k = 0; k < kSvThreads && next < 0; ++k) {
        if (segs[k] > 0.f) last_pos = k;
        if (run + segs[k] > target) {
          const int e0 = cv0 + k * kSvSeg, e1 = min(V, e0 + kSvSeg);
          for (int v = e0; v < e1; ++v) {
            const float wv = draw_weight(zrow, yrow, inv_t, lz, ly, v, mode);
            run += wv;
            if (wv > 0.f && run > target) {
              next = v;
              break;
            }
          }
          if (next < 0) {   // rounding left no crossing in this segment: take its last positive entry
            for (int v = e1 - 1; v >= e0; --v)
              if (draw_weight(zrow, yrow, inv_t, lz, ly, v, mode) > 0.f) {
                next = v;
                break;
              }
          }
          break;
        }
        run += segs[k];
      }
      if (next < 0 && last_pos >= 0) {
        // the running sum never crossed (rounding at the very end): the chunk's last positive entry
        const int e0 = cv0 + last_pos * kSvSeg, e1 = min(V, e0 + kSvSeg);
        for (int v = e1 - 1; v >= e0; --v)
          if (draw_weight(zrow, yrow, inv_t, lz, ly, v, mode) > 0.f) {
            next = v;
            break;
          }
      }
    }
  } else if (threadIdx.x == 0) {
    // a zero residual (p_a == q_{a+1} at every entry): draw from p_a over the whole row
    float tot1 = 0.f;
    for (int v = 0; v < V; ++v) tot1 += draw_weight(zrow, yrow, inv_t, lz, ly, v, 1);
    const float target = __ldg(u_final + b) * tot1;
    float run = 0.f;
    for (int v = 0; v < V && next < 0; ++v) {
      run += draw_weight(zrow, yrow, inv_t, lz, ly, v, 1);
      if (run > target) next = v;
    }
    if (next < 0) next = V - 1;
  }
  if (threadIdx.x == 0) {
    accepted[b] = a;
    next_token[b] = next < 0 ? 0 : next;
    tickets[b] = 0;
  }
}

}  // namespace dfl

namespace {
size_t sv_chunks(int V) { return (size_t)((V + dfl::kSvChunk - 1) / dfl::kSvChunk); }
}  // namespace

extern "C" size_t dflash_verify_sampled_workspace_size(int bs, int B, int V) {
  if (bs <= 0 || B <= 0 || V <= 0) return 0;
  const size_t nch = sv_chunks(V);
  const size_t stats = (size_t)bs * (2 * B - 1) * nch * 2 * sizeof(float);
  const size_t sums = (size_t)bs * nch * sizeof(float);
  const size_t tick = (size_t)bs * sizeof(int);
  return ((stats + 255) / 256) * 256 + ((sums + 255) / 256) * 256 + tick;
}

extern "C" dflash_status dflash_verify_sampled(const void* d_logits, dflash_dtype logits_dtype,
                                               const float* d_draft_logits, const int* d_draft, int bs, int B, int V,
                                               float temperature, const float* d_u_accept, const float* d_u_final,
                                               int* d_accepted, int* d_next_token, void* d_workspace,
                                               size_t workspace_bytes, void* stream) {
  dfl::TraceRange trace_("dflash_verify_sampled");
  if (bs <= 0 || B <= 0 || V <= 0 || !d_logits || !d_u_final || !d_accepted || !d_next_token || !d_workspace)
    return DFLASH_ERR_ARG;
  if (B > 1 && (!d_draft || !d_draft_logits || !d_u_accept)) return DFLASH_ERR_ARG;
  if (!(temperature > 0.f) || !std::isfinite(temperature)) return DFLASH_ERR_ARG;
  if (logits_dtype != DFLASH_F32 && logits_dtype != DFLASH_BF16) return DFLASH_ERR_ARG;
  if (workspace_bytes < dflash_verify_sampled_workspace_size(bs, B, V)) return DFLASH_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(d_workspace) & 255) != 0) return DFLASH_ERR_ARG;
  if (bs > 65535 || 2 * B - 1 > 65535) return DFLASH_ERR_UNSUPPORTED;
  const size_t nch = sv_chunks(V);
  char* ws = reinterpret_cast<char*>(d_workspace);
  float* stats = reinterpret_cast<float*>(ws);
  const size_t stats_b = (((size_t)bs * (2 * B - 1) * nch * 2 * sizeof(float) + 255) / 256) * 256;
  float* sums = reinterpret_cast<float*>(ws + stats_b);
  int* tickets = reinterpret_cast<int*>(ws + stats_b + (((size_t)bs * nch * sizeof(float) + 255) / 256) * 256);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float inv_t = 1.0f / temperature;
  const dim3 g1((unsigned)nch, (unsigned)(2 * B - 1), (unsigned)bs), g2((unsigned)nch, (unsigned)bs);
  cudaError_t e;
  if (logits_dtype == DFLASH_BF16) {
    auto Z = (const __nv_bfloat16*)d_logits;
    dfl::sv_stats_kernel<__nv_bfloat16><<<g1, dfl::kSvThreads, 0, st>>>(Z, d_draft_logits, B, V, inv_t, stats);
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = dfl::launch_kernel(dfl::sv_decide_kernel<__nv_bfloat16>, g2, dim3(dfl::kSvThreads), 0, st, true, Z,
                             d_draft_logits, d_draft, B, V, inv_t, d_u_accept, d_u_final, (const float*)stats, sums,
                             tickets, d_accepted, d_next_token);
  } else {
    auto Z = (const float*)d_logits;
    dfl::sv_stats_kernel<float><<<g1, dfl::kSvThreads, 0, st>>>(Z, d_draft_logits, B, V, inv_t, stats);
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = dfl::launch_kernel(dfl::sv_decide_kernel<float>, g2, dim3(dfl::kSvThreads), 0, st, true, Z, d_draft_logits,
                             d_draft, B, V, inv_t, d_u_accept, d_u_final, (const float*)stats, sums, tickets,
                             d_accepted, d_next_token);
  }
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ERR_CUDA;
}
