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

// RMSNorm of one fp32 row held in x_row, written to h_row (and y_row if given).
template <typename HT>
__device__ __forceinline__ void norm_row(const float* x_row, int H, const float* gain, float eps, HT* h_row,
                                         float* y_row, float* red) {
  float ss = 0.f;
  for (int c = threadIdx.x; c < H; c += blockDim.x) ss = fmaf(x_row[c], x_row[c], ss);
  ss = block_sum(ss, red);
  const float rstd = rsqrtf(ss / (float)H + eps);
  for (int c = threadIdx.x; c < H; c += blockDim.x) {
    const float y = x_row[c] * rstd * gain[c];
    h_row[c] = from_f32<HT>(y);
    if (y_row) y_row[c] = y;
  }
}

template <typename ET, typename HT>
__global__ void __launch_bounds__(kNormThreads) embed_norm_kernel(const ET* embed, const int* anchor, int mask_id,
                                                                  int B, int V, int H, const float* gain,
                                                                  float eps, float* x, HT* h, int* status) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  int tok = (m % B) == 0 ? anchor[m / B] : mask_id;
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) flag_error(status, ST_BAD_TOKEN);
    tok = 0;
  }
  float* xr = x + (size_t)m * H;
  for (int c = threadIdx.x; c < H; c += blockDim.x) xr[c] = to_f32(embed[(size_t)tok * H + c]);
  __syncthreads();
  norm_row(xr, H, gain, eps, h + (size_t)m * H, nullptr, red);
}

template <typename HT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const float* x, int H, const float* gain, float eps,
                                                               HT* h, float* y) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  norm_row(x + (size_t)m * H, H, gain, eps, h + (size_t)m * H, y ? y + (size_t)m * H : nullptr, red);
}

__global__ void argmax_finalize_kernel(unsigned long long* keys, int bs, int B, int* draft) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= bs * B) return;
  const int b = e / B, i = e % B;
  const unsigned long long k = keys[e];
  if (i > 0) draft[b * (B - 1) + i - 1] = argmax_key_index(k);
  keys[e] = 0ull;
}

void launch_embed_norm(const void* embed, int embed_bf16, const int* anchor, int mask_id, int B, int R, int V,
                       int H, const float* gain, float eps, float* x, void* h, int h_bf16, int* status,
                       cudaStream_t st) {
  if (embed_bf16 && h_bf16)
    embed_norm_kernel<__nv_bfloat16, __nv_bfloat16><<<R, kNormThreads, 0, st>>>(
        (const __nv_bfloat16*)embed, anchor, mask_id, B, V, H, gain, eps, x, (__nv_bfloat16*)h, status);
  else if (!embed_bf16 && !h_bf16)
    embed_norm_kernel<float, float><<<R, kNormThreads, 0, st>>>((const float*)embed, anchor, mask_id, B, V, H, gain,
                                                                eps, x, (float*)h, status);
  else if (embed_bf16)
    embed_norm_kernel<__nv_bfloat16, float><<<R, kNormThreads, 0, st>>>(
        (const __nv_bfloat16*)embed, anchor, mask_id, B, V, H, gain, eps, x, (float*)h, status);
  else
    embed_norm_kernel<float, __nv_bfloat16><<<R, kNormThreads, 0, st>>>(
        (const float*)embed, anchor, mask_id, B, V, H, gain, eps, x, (__nv_bfloat16*)h, status);
}

void launch_rmsnorm(const float* x, int R, int H, const float* gain, float eps, void* h, int h_bf16, float* y,
                    cudaStream_t st) {
  if (h_bf16)
    rmsnorm_kernel<__nv_bfloat16><<<R, kNormThreads, 0, st>>>(x, H, gain, eps, (__nv_bfloat16*)h, y);
  else
    rmsnorm_kernel<float><<<R, kNormThreads, 0, st>>>(x, H, gain, eps, (float*)h, y);
}

void launch_argmax_finalize(unsigned long long* keys, int bs, int B, int* draft, cudaStream_t st) {
  const int n = bs * B;
  argmax_finalize_kernel<<<(n + 255) / 256, 256, 0, st>>>(keys, bs, B, draft);
}

}  // namespace dfl
