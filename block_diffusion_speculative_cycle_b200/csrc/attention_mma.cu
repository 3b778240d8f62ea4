// Tensor-core block attention (bf16 in, fp32 accumulate) for the drafter.
//
// One CTA per (split of the key range, KV head, request); the splits of one
// (request, KV head) form a thread-block cluster. The g*B block queries
// of the head group (g = n_q/n_kv query heads x B block rows, <= 128 rows) are
// split into 16-row slices, one per warp, held as mma.sync A fragments. Keys
// stream through shared memory in tiles of 64 (a ring of 2-3 stages, cp.async 16-byte
// copies, XOR-swizzled rows so ldmatrix is conflict-free): context keys come
// from the request's cache pages, the B block keys from the block K/V rows.
// Per tile: S = Q·Kᵀ (m16n8k16), online softmax in fp32 (exp2 domain, quad
// shuffles), O += P·V with P re-packed from the S accumulators. The split's
// state (unnormalised O, running max m, sum l) is staged in shared memory; after a
// cluster barrier each CTA combines a share of the rows over all splits through
// distributed shared memory (log-sum-exp weights, split order) and writes them.
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace dfl {

namespace {

constexpr int kKT = 64;   // keys per tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Element offset of (row, 8-wide chunk) in a [rows][D] bf16 tile with the
// 16-byte chunks of each row XOR-swizzled by row % 8.
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

}  // namespace

// Stages of the K/V ring: 3 for up to 64 query rows, 2 for 128 (both fit two CTAs per SM).
template <int D, int NST>
__global__ void __launch_bounds__(256) attn_cluster_kernel(const AttnParams p, __nv_bfloat16* out) {
  constexpr int CH = D / 8;    // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int nr = p.g * p.B;
  const int rows_pad = ((nr + 15) / 16) * 16;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);   // [rows_pad][D]
  __nv_bfloat16* ring = qs + rows_pad * D;                           // NST x ([kKT][D] K, [kKT][D] V)
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int q_dim = p.n_q * D, kv_dim = p.n_kv * D;
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.kblk);
  const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(p.vblk);
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.kc);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.vc);
  grid_dep_wait();
  grid_dep_launch();

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (tid == 0) flag_error(p.status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  const int T_all = P + p.B;
  const int k0 = s * p.kps, k1 = min(T_all, k0 + p.kps);
  const int n_tiles = k1 > k0 ? (k1 - k0 + kKT - 1) / kKT : 0;

  auto load_tile = [&](int kt, int stage) {
    __nv_bfloat16* kd = ring + stage * 2 * kKT * D;
    __nv_bfloat16* vd = kd + kKT * D;
    for (int e = tid; e < kKT * CH; e += nthr) {
      const int r = e / CH, c = e % CH, key = kt + r;
      const __nv_bfloat16* ksrc = kb;
      const __nv_bfloat16* vsrc = vb;
      int bytes = 0;
      if (key < k1) {
        if (key < P) {
          const int slot = key / p.page_size;
          const int page = slot < p.max_pages ? p.page_table[(size_t)b * p.max_pages + slot] : -1;
          if (page >= 0 && page < p.num_pages) {
            const size_t off = (((size_t)page * p.n_kv + h) * p.page_size + key % p.page_size) * D + c * 8;
            ksrc = kc + off;
            vsrc = vc + off;
            bytes = 16;
          } else if (c == 0) {
            flag_error(p.status, ST_BAD_PAGE);
          }
        } else {
          const size_t off = (size_t)(b * p.B + key - P) * kv_dim + h * D + c * 8;
          ksrc = kb + off;
          vsrc = vb + off;
          bytes = 16;
        }
      }
      cp_async16(kd + swz<D>(r, c), ksrc, bytes);
      cp_async16(vd + swz<D>(r, c), vsrc, bytes);
    }
  };

  // group 0: Q rows (r = j*B + i: query head h*g + j, block row i) and tile 0; groups 1..NST-1: tiles 1..
  for (int e = tid; e < rows_pad * CH; e += nthr) {
    const int r = e / CH, c = e % CH;
    const __nv_bfloat16* src = q;
    int bytes = 0;
    if (r < nr) {
      const int j = r / p.B, i = r % p.B;
      src = q + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + c * 8;
      bytes = 16;
    }
    cp_async16(qs + swz<D>(r, c), src, bytes);
  }
#pragma unroll
  for (int i = 0; i < NST; ++i) {
    if (i < n_tiles) load_tile(k0 + i * kKT, i);
    cp_async_commit();
  }

  const bool active = warp * 16 < nr;
  uint32_t qf[D / 16][4];
  const float sl2 = p.scale * 1.4426950408889634f;   // softmax in the exp2 domain
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows gid, gid+8 of this warp
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  for (int t = 0; t < n_tiles; ++t) {
    cp_async_wait<NST - 1>();   // tile t (and Q) have landed
    __syncthreads();
    if (active) {
      if (t == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int mat = lane >> 3, r = lane & 7;
          ldsm_x4(qf[kk], qs + swz<D>(warp * 16 + r + 8 * (mat & 1), 2 * kk + (mat >> 1)));
        }
      }
      const int kt = k0 + t * kKT;
      const __nv_bfloat16* kt_s = ring + (t % NST) * 2 * kKT * D;
      const __nv_bfloat16* vt_s = kt_s + kKT * D;
      float sc[kKT / 8][4];
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int n = 0; n < kKT / 8; n += 2) {
          const int mat = lane >> 3, r = lane & 7;
          uint32_t bfr[4];
          ldsm_x4(bfr, kt_s + swz<D>(n * 8 + r + 8 * (mat >> 1), 2 * kk + (mat & 1)));
          mma_16816(sc[n], qf[kk], bfr[0], bfr[1]);
          mma_16816(sc[n + 1], qf[kk], bfr[2], bfr[3]);
        }
      }
      float mx0 = m0, mx1 = m1;
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) {
        const int key = kt + n * 8 + 2 * tig;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const bool ok = key + c < k1;
          sc[n][c] = ok ? sc[n][c] * sl2 : -INFINITY;
          sc[n][2 + c] = ok ? sc[n][2 + c] * sl2 : -INFINITY;
          mx0 = fmaxf(mx0, sc[n][c]);
          mx1 = fmaxf(mx1, sc[n][2 + c]);
        }
      }
#pragma unroll
      for (int m = 1; m <= 2; m <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, m));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, m));
      }
      const float a0 = exp2f(m0 - mx0), a1 = exp2f(m1 - mx1);
      m0 = mx0;
      m1 = mx1;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pf[kKT / 16][4];
#pragma unroll
      for (int n = 0; n < kKT / 8; ++n) {
        const float p00 = exp2f(sc[n][0] - m0), p01 = exp2f(sc[n][1] - m0);
        const float p10 = exp2f(sc[n][2] - m1), p11 = exp2f(sc[n][3] - m1);
        rs0 += p00 + p01;
        rs1 += p10 + p11;
        pf[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p00, p01);
        pf[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p10, p11);
      }
      l0 = l0 * a0 + rs0;
      l1 = l1 * a1 + rs1;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        o[n][0] *= a0;
        o[n][1] *= a0;
        o[n][2] *= a1;
        o[n][3] *= a1;
      }
#pragma unroll
      for (int kk = 0; kk < kKT / 16; ++kk) {
#pragma unroll
        for (int n = 0; n < D / 8; n += 2) {
          const int mat = lane >> 3, r = lane & 7;
          uint32_t bfr[4];
          ldsm_x4_t(bfr, vt_s + swz<D>(kk * 16 + r + 8 * (mat & 1), n + (mat >> 1)));
          mma_16816(o[n], pf[kk], bfr[0], bfr[1]);
          mma_16816(o[n + 1], pf[kk], bfr[2], bfr[3]);
        }
      }
    }
    __syncthreads();   // stage t % NST is free again
    if (t + NST < n_tiles) load_tile(k0 + (t + NST) * kKT, t % NST);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();   // every copy has landed and every warp is done with the ring

  if (active) {
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, m);
      l1 += __shfl_xor_sync(0xffffffffu, l1, m);
    }
  }
  const int r0 = warp * 16 + gid, r1 = r0 + 8;
  const int S = p.n_splits;
  if (S == 1) {
    // the whole key range is here: normalise and write
    if (active) {
      const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        const int d = n * 8 + 2 * tig;
        if (r0 < nr) {
          const int j = r0 / p.B, i = r0 % p.B;
          *reinterpret_cast<__nv_bfloat162*>(out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + d) =
              __floats2bfloat162_rn(o[n][0] * i0, o[n][1] * i0);
        }
        if (r1 < nr) {
          const int j = r1 / p.B, i = r1 % p.B;
          *reinterpret_cast<__nv_bfloat162*>(out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + d) =
              __floats2bfloat162_rn(o[n][2] * i1, o[n][3] * i1);
        }
      }
    }
    return;
  }

  // ---- cluster merge: stage (O, m, l) of this split, then CTA `rank` combines its share of rows
  float* so = reinterpret_cast<float*>(smem_raw);   // [nr][D] unnormalised O
  float* sm = so + nr * D;                          // [nr] running max (exp2 domain)
  float* sl = sm + nr;                              // [nr] running sum
  if (active) {
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int d = n * 8 + 2 * tig;
      if (r0 < nr) *reinterpret_cast<float2*>(so + r0 * D + d) = make_float2(o[n][0], o[n][1]);
      if (r1 < nr) *reinterpret_cast<float2*>(so + r1 * D + d) = make_float2(o[n][2], o[n][3]);
    }
    if (tig == 0) {
      if (r0 < nr) {
        sm[r0] = m0;
        sl[r0] = l0;
      }
      if (r1 < nr) {
        sm[r1] = m1;
        sl[r1] = l1;
      }
    }
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  const int per = (nr + S - 1) / S;
  const int lo = s * per, hi = min(nr, lo + per);
  const int nwarps = nthr >> 5;
  for (int r = lo + warp; r < hi; r += nwarps) {
    // lanes own splits for the max and the weights
    float ms = -INFINITY, ls = 0.f;
    if (lane < S) {
      const float* rsm = cluster.map_shared_rank(sm, lane);
      const float* rsl = cluster.map_shared_rank(sl, lane);
      ms = rsm[r];
      ls = rsl[r];
    }
    float M = ms;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    const float w = lane < S ? exp2f(ms - M) : 0.f;
    float L = ls * w;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) L += __shfl_xor_sync(0xffffffffu, L, m);
    const float invL = 1.f / L;
    float acc[D / 32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
    for (int k = 0; k < S; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float* ro = cluster.map_shared_rank(so, k) + r * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(wk, ro[lane + 32 * c], acc[c]);
    }
    const int j = r / p.B, i = r % p.B;
    __nv_bfloat16* dst = out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) dst[lane + 32 * c] = __float2bfloat16_rn(acc[c] * invL);
  }
  cluster.sync();   // peers may still be reading this CTA's staging
}

static size_t attn_cluster_smem(int d, int rows_pad, int nst) {
  const size_t loads = ((size_t)rows_pad + (size_t)nst * 2 * kKT) * d * 2;
  const size_t merge = ((size_t)rows_pad * d + 2 * rows_pad) * 4;
  return loads > merge ? loads : merge;
}

template <int D, int NST>
static cudaError_t launch_cluster_t(const AttnParams& p, void* out, cudaStream_t st, bool pdl) {
  const int nr = p.g * p.B;
  const int rows_pad = ((nr + 15) / 16) * 16;
  const int warps = rows_pad / 16;
  const int threads = 32 * (warps < 4 ? 4 : warps);
  const size_t smem = attn_cluster_smem(D, rows_pad, NST);
  static size_t set = 0;
  if (smem > set) {
    cudaError_t e = cudaFuncSetAttribute(attn_cluster_kernel<D, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_cluster_kernel<D, NST>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    set = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, p.n_kv, p.bs);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.n_splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.n_splits > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_cluster_kernel<D, NST>, p, (__nv_bfloat16*)out);
}

cudaError_t launch_attn_cluster(const AttnParams& p, void* out, cudaStream_t st, bool pdl) {
  if (p.n_splits < 1 || p.n_splits > kMaxAttnCluster || p.kps % kKT) return cudaErrorInvalidValue;
  const bool wide = p.g * p.B > 64;
  if (p.d == 128) return wide ? launch_cluster_t<128, 2>(p, out, st, pdl) : launch_cluster_t<128, 3>(p, out, st, pdl);
  return wide ? launch_cluster_t<64, 2>(p, out, st, pdl) : launch_cluster_t<64, 3>(p, out, st, pdl);
}

}  // namespace dfl
