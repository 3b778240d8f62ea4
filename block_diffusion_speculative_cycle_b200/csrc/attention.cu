// Block attention of the drafter: for request b and KV head h, the g*B block
// queries of that head group attend to the request's injected context keys
// (positions 0..P-1, read through the page table) and to all B block keys,
// with no mask (in-block attention is non-causal). The key range is split
// across CTAs; each split keeps an online-softmax state (running max m, sum l,
// unnormalised output o) in fp32, and a merge kernel combines the splits with
// log-sum-exp weights.
#include "kernels.cuh"

namespace dfl {

constexpr int kAttnThreads = 256;
constexpr int kKeyTile = 32;

template <typename T, int D, int RPW>
__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(const AttnParams p) {
  extern __shared__ float sm[];
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nr = p.g * p.B;
  const int q_dim = p.n_q * D, kv_dim = p.n_kv * D;
  float* qs = sm;                          // [nr][D]
  float* ks = qs + nr * D;                 // [kKeyTile][D+1]
  float* vs = ks + kKeyTile * (D + 1);     // [kKeyTile][D+1]
  const T* q = reinterpret_cast<const T*>(p.q);
  const T* kb = reinterpret_cast<const T*>(p.kblk);
  const T* vb = reinterpret_cast<const T*>(p.vblk);
  const T* kc = reinterpret_cast<const T*>(p.kc);
  const T* vc = reinterpret_cast<const T*>(p.vc);
  grid_dep_wait();
  grid_dep_launch();

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (threadIdx.x == 0) flag_error(p.status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  const int T_all = P + p.B;
  const int ctx_lo = attn_ctx_lo(P, p.window);
  const int k0 = min(T_all, attn_key_base(ctx_lo) + s * p.kps),
            k1 = s == p.n_splits - 1 ? T_all : min(T_all, k0 + p.kps);

  for (int e = threadIdx.x; e < nr * D; e += kAttnThreads) {
    const int r = e / D, dd = e % D, j = r / p.B, i = r % p.B;
    qs[e] = to_f32(q[(size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + dd]) * p.scale;
  }
  float m[RPW], l[RPW], o[RPW][D / 32];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[rr][c] = 0.f;
  }
  __syncthreads();

  for (int kt = k0; kt < k1; kt += kKeyTile) {
    for (int e = threadIdx.x; e < kKeyTile * D; e += kAttnThreads) {
      const int kk = e / D, dd = e % D, key = kt + kk;
      float kv = 0.f, vv = 0.f;
      if (key < k1 && key >= ctx_lo) {
        if (key < P) {
          const int slot = key / p.page_size;
          const int page = slot < p.max_pages ? p.page_table[(size_t)b * p.max_pages + slot] : -1;
          if (page >= 0 && page < p.num_pages) {
            const size_t idx = (((size_t)page * p.n_kv + h) * p.page_size + key % p.page_size) * D + dd;
            kv = to_f32(kc[idx]);
            vv = to_f32(vc[idx]);
          } else if (dd == 0) {
            flag_error(p.status, ST_BAD_PAGE);
          }
        } else {
          const size_t idx = (size_t)(b * p.B + key - P) * kv_dim + h * D + dd;
          kv = to_f32(kb[idx]);
          vv = to_f32(vb[idx]);
        }
      }
      ks[kk * (D + 1) + dd] = kv;
      vs[kk * (D + 1) + dd] = vv;
    }
    __syncthreads();
    const bool valid = kt + lane < k1 && kt + lane >= ctx_lo;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int r = warp + 8 * rr;
      if (r < nr) {
        float sc = -INFINITY;
        // a causal decoder's row i (position P + i) sees block keys 0..i only
        if (valid && !(p.causal && kt + lane >= P && kt + lane - P > r % p.B)) {
          float dot = 0.f;
#pragma unroll 8
          for (int dd = 0; dd < D; ++dd) dot = fmaf(qs[r * D + dd], ks[lane * (D + 1) + dd], dot);
          sc = dot;
        }
        const float mn = fmaxf(m[rr], warp_max(sc));
        const float pe = sc != -INFINITY ? expf(sc - mn) : 0.f;
        // a tile with every key masked (below a sliding window's start) while the
        // row has seen no key yet leaves the state as it is
        const float alpha = mn == -INFINITY ? 1.f : expf(m[rr] - mn);
        l[rr] = l[rr] * alpha + warp_sum(pe);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) o[rr][c] *= alpha;
#pragma unroll 4
        for (int kk = 0; kk < kKeyTile; ++kk) {
          const float pk = __shfl_sync(0xffffffffu, pe, kk);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) o[rr][c] = fmaf(pk, vs[kk * (D + 1) + lane + 32 * c], o[rr][c]);
        }
        m[rr] = mn;
      }
    }
    __syncthreads();
  }

  const size_t pbase = ((size_t)(b * p.n_kv + h) * p.n_splits + s) * nr;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = warp + 8 * rr;
    if (r < nr) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) p.part_o[(pbase + r) * D + lane + 32 * c] = o[rr][c];
      if (lane == 0) {
        p.part_m[pbase + r] = m[rr];
        p.part_l[pbase + r] = l[rr];
      }
    }
  }
}

// One warp per (block row, query head): merge the splits that hold keys. Lanes
// own splits for the max and the weights; the weighted sum of the split outputs
// then reads each split's row with all lanes (d/32 values per lane).
template <typename OT, int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnParams p, OT* out) {
  grid_dep_wait();
  grid_dep_launch();
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int R = p.bs * p.B;
  if (gw >= R * p.n_q) return;
  const int m_row = gw / p.n_q, j = gw % p.n_q;
  const int b = m_row / p.B, i = m_row % p.B;
  const int h = j / p.g, jj = j % p.g;
  const int nr = p.g * p.B, r = jj * p.B + i;
  int P = p.ctx_len[b];
  P = P < 0 ? 0 : (P > p.max_ctx ? p.max_ctx : P);
  const int used = min(p.n_splits, (P + p.B - attn_key_base(attn_ctx_lo(P, p.window)) + p.kps - 1) / p.kps);
  const size_t base = (size_t)(b * p.n_kv + h) * p.n_splits * nr + r;
  float M = -INFINITY;
  for (int s = lane; s < used; s += 32) M = fmaxf(M, p.part_m[base + (size_t)s * nr]);
  M = warp_max(M);
  float L = 0.f;
  for (int s = lane; s < used; s += 32) {
    const size_t idx = base + (size_t)s * nr;
    L += p.part_l[idx] * expf(p.part_m[idx] - M);
  }
  L = warp_sum(L);
  const float invL = 1.f / L;
  float acc[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
  for (int s0 = 0; s0 < used; s0 += 32) {
    const int sl = s0 + lane;
    const float wl = sl < used ? expf(p.part_m[base + (size_t)sl * nr] - M) * invL : 0.f;
    const int n = min(32, used - s0);
#pragma unroll 4
    for (int k = 0; k < n; ++k) {
      const float w = __shfl_sync(0xffffffffu, wl, k);
      const float* o = p.part_o + (base + (size_t)(s0 + k) * nr) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(w, o[lane + 32 * c], acc[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < D / 32; ++c) out[(size_t)m_row * p.n_q * D + j * D + lane + 32 * c] = from_f32<OT>(acc[c]);
}

template <typename T, int D, int RPW>
static cudaError_t launch_split(const AttnParams& p, cudaStream_t st, bool pdl) {
  const int nr = p.g * p.B;
  const size_t smem = ((size_t)nr * D + 2 * kKeyTile * (D + 1)) * sizeof(float);
  static size_t attr_bytes = 0;
  if (smem > attr_bytes) {
    cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<T, D, RPW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes = smem;
  }
  return launch_kernel(attn_split_kernel<T, D, RPW>, dim3(p.n_splits, p.n_kv, p.bs), dim3(kAttnThreads), smem, st,
                       pdl, p);
}

template <typename T, int D>
static cudaError_t launch_split_rpw(const AttnParams& p, cudaStream_t st, bool pdl) {
  const int rpw = (p.g * p.B + 7) / 8;
  if (rpw <= 1) return launch_split<T, D, 1>(p, st, pdl);
  if (rpw <= 2) return launch_split<T, D, 2>(p, st, pdl);
  if (rpw <= 4) return launch_split<T, D, 4>(p, st, pdl);
  if (rpw <= 8) return launch_split<T, D, 8>(p, st, pdl);
  return launch_split<T, D, 16>(p, st, pdl);
}

cudaError_t launch_attention(const AttnParams& p, void* out, int out_bf16, int in_bf16, cudaStream_t st, bool pdl) {
  if (in_bf16 && out_bf16) return launch_attn_cluster(p, out, st, pdl);
  cudaError_t e = p.d == 128 ? launch_split_rpw<float, 128>(p, st, pdl) : launch_split_rpw<float, 64>(p, st, pdl);
  if (e != cudaSuccess) return e;
  const int warps = p.bs * p.B * p.n_q;
  const dim3 grid((warps + 7) / 8), block(256);
  if (p.d == 128) return launch_kernel(attn_merge_kernel<float, 128>, grid, block, 0, st, pdl, p, (float*)out);
  return launch_kernel(attn_merge_kernel<float, 64>, grid, block, 0, st, pdl, p, (float*)out);
}

}  // namespace dfl
