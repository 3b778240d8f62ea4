// Embedding gather, RMSNorm and the argmax finalisation of the draft pass.
#include "kernels.cuh"

namespace dfl {

constexpr int kNormThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  if (warp == 0) {
    t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}

// Load x[0..H) (fp32) into registers as float4, VPT per thread; returns the sum of squares.
template <int VPT>
__device__ __forceinline__ float load_row(const float* x_row, int H, float4* v) {
  const float4* xr = reinterpret_cast<const float4*>(x_row);
  const int n4 = H >> 2;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * blockDim.x + threadIdx.x;
    v[i] = idx < n4 ? xr[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i) ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  return ss;
}

__device__ __forceinline__ void store4(float* dst, float4 v, size_t = 0) { *reinterpret_cast<float4*>(dst) = v; }
// bf16 rows; with plane != 0 also the lo plane bf16(v - hi) `plane` elements on
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v, size_t plane = 0) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
  if (plane) {
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    __nv_bfloat162 la = __floats2bfloat162_rn(v.x - fa.x, v.y - fa.y), lb = __floats2bfloat162_rn(v.z - fb.x, v.w - fb.y);
    u.x = *reinterpret_cast<uint32_t*>(&la);
    u.y = *reinterpret_cast<uint32_t*>(&lb);
    *reinterpret_cast<uint2*>(dst + plane) = u;
  }
}

// h = v * rsqrt(ss/H + eps) * gain (h and/or an fp32 copy y, each if given)
template <int VPT, typename HT>
__device__ __forceinline__ void norm_store(const float4* v, float ss, int H, const float* gain, float eps, HT* h_row,
                                           float* y_row, float* red, size_t h_plane = 0) {
  ss = block_sum(ss, red);
  const float rstd = rsqrtf(ss / (float)H + eps);
  const float4* g4 = reinterpret_cast<const float4*>(gain);
  const int n4 = H >> 2;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * blockDim.x + threadIdx.x;
    if (idx < n4) {
      const float4 g = g4[idx];
      const float4 y = make_float4(v[i].x * rstd * g.x, v[i].y * rstd * g.y, v[i].z * rstd * g.z, v[i].w * rstd * g.w);
      if (h_row) store4(h_row + 4 * idx, y, h_plane);
      if (y_row) store4(y_row + 4 * idx, y);
    }
  }
}

template <int VPT, typename ET, typename HT>
__global__ void __launch_bounds__(kNormThreads) embed_norm_kernel(const ET* embed, const int* anchor, int mask_id,
                                                                  const int* tokens, const int* draft, int B, int V,
                                                                  int H, const float* gain, float eps, float* x, HT* h,
                                                                  size_t h_plane, int* status, const RopeFill rf,
                                                                  const AttnKpsPlan kp) {
  __shared__ float red[32];
  grid_dep_wait();
  grid_dep_launch();
  const int m = blockIdx.x;
  if (kp.out && m == 0 && threadIdx.x < 32) {
    // the attention split size of this call (AttnKpsPlan), one warp
    const int lane = threadIdx.x;
    auto tiles_of = [&](int r) {
      int P = kp.ctx_len[r];
      P = P < 0 ? 0 : (P > kp.max_ctx ? kp.max_ctx : P);
      return (P + kp.B - attn_key_base(attn_ctx_lo(P, kp.window)) + 63) / 64;
    };
    int sum_t = 0, max_t = 0;
    for (int r = lane; r < kp.bs; r += 32) {
      const int t = tiles_of(r);
      sum_t += t;
      max_t = max(max_t, t);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum_t += __shfl_xor_sync(0xffffffffu, sum_t, o);
      max_t = max(max_t, __shfl_xor_sync(0xffffffffu, max_t, o));
    }
    const int per_head = max(1, kp.slots / kp.n_kv);
    long long best_cost = -1;
    int best = max(kp.min_tiles, max_t), best_items = 0;
    for (int cand = 0; cand < 20; ++cand) {
      int c = cand < 16 ? (max_t + cand) / (cand + 1) : (sum_t + (cand - 15) * per_head - 1) / ((cand - 15) * per_head);
      c = max(kp.min_tiles, max(1, c));
      int items = 0;
      for (int r = lane; r < kp.bs; r += 32) items += (tiles_of(r) + c - 1) / c;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) items += __shfl_xor_sync(0xffffffffu, items, o);
      const long long waves = ((long long)items * kp.n_kv + kp.slots - 1) / kp.slots;
      const long long cost = waves * (kAttnPlanStartTiles + c);
      if (best_cost < 0 || cost < best_cost || (cost == best_cost && c > best)) {
        best_cost = cost;
        best = c;
        best_items = items;
      }
    }
    if (lane == 0) {
      kp.out[0] = 64 * best;   // keys per split
      kp.out[1] = best_items;  // (request, split) items of the batch
    }
  }
  // this row's entries of the call's RoPE table (read by the QKV epilogues)
  if (rf.out)
    for (int i = threadIdx.x; i < rf.half; i += blockDim.x) rope_fill_entry(rf, m * rf.half + i);
  // row (request m / B, position m % B): tokens[m] when given; else the anchor at
  // position 0 and, at positions i >= 1, draft[request, i-1] (given) or the mask id
  const int i = m % B;
  int tok = tokens ? tokens[m] : (i == 0 ? anchor[m / B] : (draft ? draft[(size_t)(m / B) * (B - 1) + i - 1] : mask_id));
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) flag_error(status, ST_BAD_TOKEN);
    tok = 0;
  }
  const ET* er = embed + (size_t)tok * H;
  float4 v[VPT];
  float ss = 0.f;
  const int n4 = H >> 2;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * blockDim.x + threadIdx.x;
    v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (idx < n4)
      v[i] = make_float4(to_f32(er[4 * idx]), to_f32(er[4 * idx + 1]), to_f32(er[4 * idx + 2]), to_f32(er[4 * idx + 3]));
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * blockDim.x + threadIdx.x;
    if (idx < n4) store4(x + (size_t)m * H + 4 * idx, v[i]);
    ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  }
  norm_store<VPT>(v, ss, H, gain, eps, h + (size_t)m * H, nullptr, red, h_plane);
}

template <int VPT, typename HT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const float* x, int H, const float* gain, float eps,
                                                               HT* h, float* y) {
  __shared__ float red[32];
  grid_dep_wait();
  grid_dep_launch();
  const int m = blockIdx.x;
  float4 v[VPT];
  const float ss = load_row<VPT>(x + (size_t)m * H, H, v);
  norm_store<VPT>(v, ss, H, gain, eps, h ? h + (size_t)m * H : nullptr, y ? y + (size_t)m * H : nullptr, red);
}

__global__ void argmax_finalize_kernel(unsigned long long* keys, int bs, int B, int* draft) {
  grid_dep_wait();
  grid_dep_launch();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= bs * B) return;
  const int b = e / B, i = e % B;
  const unsigned long long k = keys[e];
  if (i > 0) draft[b * (B - 1) + i - 1] = argmax_key_index(k);
  keys[e] = 0ull;
}

template <int VPT>
static cudaError_t embed_norm_vpt(const void* embed, int embed_bf16, const int* anchor, int mask_id,
                                  const int* tokens, const int* draft, int B, int R, int V, int H, const float* gain, float eps, float* x, void* h, int h_bf16,
                                  size_t h_plane, int* status, const RopeFill& rf, const AttnKpsPlan& kp,
                                  cudaStream_t st, bool pdl) {
  const dim3 g(R), b(kNormThreads);
  if (embed_bf16 && h_bf16)
    return launch_kernel(embed_norm_kernel<VPT, __nv_bfloat16, __nv_bfloat16>, g, b, 0, st, pdl,
                         (const __nv_bfloat16*)embed, anchor, mask_id, tokens, draft, B, V, H, gain, eps, x, (__nv_bfloat16*)h,
                         h_plane, status, rf, kp);
  if (!embed_bf16 && !h_bf16)
    return launch_kernel(embed_norm_kernel<VPT, float, float>, g, b, 0, st, pdl, (const float*)embed, anchor,
                         mask_id, tokens, draft, B, V, H, gain, eps, x, (float*)h, (size_t)0, status, rf, kp);
  if (embed_bf16)
    return launch_kernel(embed_norm_kernel<VPT, __nv_bfloat16, float>, g, b, 0, st, pdl,
                         (const __nv_bfloat16*)embed, anchor, mask_id, tokens, draft, B, V, H, gain, eps, x, (float*)h, (size_t)0,
                         status, rf, kp);
  return launch_kernel(embed_norm_kernel<VPT, float, __nv_bfloat16>, g, b, 0, st, pdl, (const float*)embed, anchor,
                       mask_id, tokens, draft, B, V, H, gain, eps, x, (__nv_bfloat16*)h, h_plane, status, rf, kp);
}

cudaError_t launch_embed_norm(const void* embed, int embed_bf16, const int* anchor, int mask_id, const int* tokens,
                              const int* draft, int B, int R, int V, int H, const float* gain, float eps, float* x, void* h, int h_bf16, size_t h_plane,
                              int* status, const RopeFill& rf, const AttnKpsPlan& kp, cudaStream_t st, bool pdl) {
  const int vpt = (H / 4 + kNormThreads - 1) / kNormThreads;
  if (vpt <= 1)
    return embed_norm_vpt<1>(embed, embed_bf16, anchor, mask_id, tokens, draft, B, R, V, H, gain, eps, x, h, h_bf16, h_plane, status,
                             rf, kp, st, pdl);
  if (vpt <= 2)
    return embed_norm_vpt<2>(embed, embed_bf16, anchor, mask_id, tokens, draft, B, R, V, H, gain, eps, x, h, h_bf16, h_plane, status,
                             rf, kp, st, pdl);
  if (vpt <= 4)
    return embed_norm_vpt<4>(embed, embed_bf16, anchor, mask_id, tokens, draft, B, R, V, H, gain, eps, x, h, h_bf16, h_plane, status,
                             rf, kp, st, pdl);
  return embed_norm_vpt<8>(embed, embed_bf16, anchor, mask_id, tokens, draft, B, R, V, H, gain, eps, x, h, h_bf16, h_plane, status,
                           rf, kp, st, pdl);
}

template <int VPT>
static cudaError_t rmsnorm_vpt(const float* x, int R, int H, const float* gain, float eps, void* h, int h_bf16,
                               float* y, cudaStream_t st, bool pdl) {
  if (h_bf16)
    return launch_kernel(rmsnorm_kernel<VPT, __nv_bfloat16>, dim3(R), dim3(kNormThreads), 0, st, pdl, x, H, gain,
                         eps, (__nv_bfloat16*)h, y);
  return launch_kernel(rmsnorm_kernel<VPT, float>, dim3(R), dim3(kNormThreads), 0, st, pdl, x, H, gain, eps,
                       (float*)h, y);
}

cudaError_t launch_rmsnorm(const float* x, int R, int H, const float* gain, float eps, void* h, int h_bf16, float* y,
                           cudaStream_t st, bool pdl) {
  const int vpt = (H / 4 + kNormThreads - 1) / kNormThreads;
  if (vpt <= 1) return rmsnorm_vpt<1>(x, R, H, gain, eps, h, h_bf16, y, st, pdl);
  if (vpt <= 2) return rmsnorm_vpt<2>(x, R, H, gain, eps, h, h_bf16, y, st, pdl);
  if (vpt <= 4) return rmsnorm_vpt<4>(x, R, H, gain, eps, h, h_bf16, y, st, pdl);
  return rmsnorm_vpt<8>(x, R, H, gain, eps, h, h_bf16, y, st, pdl);
}

cudaError_t launch_argmax_finalize(unsigned long long* keys, int bs, int B, int* draft, cudaStream_t st, bool pdl) {
  const int n = bs * B;
  return launch_kernel(argmax_finalize_kernel, dim3((n + 255) / 256), dim3(256), 0, st, pdl, keys, bs, B, draft);
}

}  // namespace dfl

namespace dfl {

// One block per row: copy the row's n_kv*d keys and values into its cache page.
__global__ void __launch_bounds__(128) kv_scatter_kernel(const float* kb, const float* vb, const int* pos0, int n,
                                                         int n_kv, int d, const int* page_table, int max_pages,
                                                         int num_pages, int page_size, float* kc, float* vc,
                                                         int* status) {
  grid_dep_wait();
  grid_dep_launch();
  const int m = blockIdx.x;
  const int req = m / n;
  const int pos = pos0[req] + m % n;
  const int slot = pos >= 0 ? pos / page_size : -1;
  const int page = slot >= 0 && slot < max_pages ? page_table[(size_t)req * max_pages + slot] : -1;
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) flag_error(status, ST_BAD_PAGE);
    return;
  }
  const int kvd = n_kv * d;
  for (int e = threadIdx.x; e < kvd; e += blockDim.x) {
    const int head = e / d, j = e % d;
    const size_t dst = (((size_t)page * n_kv + head) * page_size + pos % page_size) * d + j;
    kc[dst] = kb[(size_t)m * kvd + e];
    vc[dst] = vb[(size_t)m * kvd + e];
  }
}

cudaError_t launch_kv_scatter(const float* kb, const float* vb, const int* pos0, int n, int R, int n_kv, int d,
                              const int* page_table, int max_pages, int num_pages, int page_size, float* kc, float* vc,
                              int* status, cudaStream_t st) {
  return launch_kernel(kv_scatter_kernel, dim3(R), dim3(128), 0, st, true, kb, vb, pos0, n, n_kv, d, page_table,
                       max_pages, num_pages, page_size, kc, vc, status);
}

// One thread per request: commit d_1..d_a and next, then advance the request's
// state for the next cycle (anchor, context length, injection rows and start).
__global__ void spec_commit_kernel(int bs, int B, const int* draft, const int* accepted, const int* next_token,
                                   int* out_tokens, int max_out, int* out_len, int* anchor, int* ctx_len, int* n_new,
                                   int* start_pos) {
  grid_dep_wait();
  grid_dep_launch();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= bs) return;
  const int a = accepted[b], nxt = next_token[b];
  int len = out_len[b];
  int* out = out_tokens + (size_t)b * max_out;
  for (int i = 0; i < a; ++i)
    if (len < max_out) out[len++] = draft[(size_t)b * (B - 1) + i];
  if (len < max_out) out[len++] = nxt;
  out_len[b] = len;
  const int P = ctx_len[b];
  start_pos[b] = P;
  n_new[b] = a + 1;
  ctx_len[b] = P + a + 1;
  anchor[b] = nxt;
}

cudaError_t launch_spec_commit(int bs, int B, const int* draft, const int* accepted, const int* next_token,
                               int* out_tokens, int max_out, int* out_len, int* anchor, int* ctx_len, int* n_new,
                               int* start_pos, cudaStream_t st) {
  return launch_kernel(spec_commit_kernel, dim3((bs + 127) / 128), dim3(128), 0, st, true, bs, B, draft, accepted,
                       next_token, out_tokens, max_out, out_len, anchor, ctx_len, n_new, start_pos);
}

}  // namespace dfl
