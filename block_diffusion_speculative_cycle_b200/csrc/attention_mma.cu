// Tensor-core block attention (bf16 in, fp32 accumulate) for the drafter.
//
// One CTA per (split of the key range, KV head, request). The g*B block queries
// of the head group (g = n_q/n_kv query heads x B block rows, <= 128 rows) are
// split into 16-row slices, one per warp, held as mma.sync A fragments. Keys
// stream through shared memory in tiles of 64 (two buffers, cp.async 16-byte
// copies, XOR-swizzled rows so ldmatrix is conflict-free): context keys come
// from the request's cache pages, the B block keys from the block K/V rows.
// Per tile: S = Q·Kᵀ (m16n8k16), online softmax in fp32 (exp2 domain, quad
// shuffles), O += P·V with P re-packed from the S accumulators. The split's
// state (unnormalised O, running max m in natural-log units, sum l) goes to the
// partial buffers that attn_merge_kernel combines.
#include "kernels.cuh"

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

template <int D>
__global__ void __launch_bounds__(256) attn_mma_kernel(const AttnParams p) {
  constexpr int CH = D / 8;    // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);   // [128][D]
  __nv_bfloat16* ks = qs + 128 * D;                                  // [2][kKT][D]
  __nv_bfloat16* vs = ks + 2 * kKT * D;                              // [2][kKT][D]
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int nr = p.g * p.B;
  const int q_dim = p.n_q * D, kv_dim = p.n_kv * D;
  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.kblk);
  const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(p.vblk);
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.kc);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.vc);

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (tid == 0) flag_error(p.status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  const int T_all = P + p.B;
  const int k0 = s * p.kps, k1 = min(T_all, k0 + p.kps);
  const int n_tiles = k1 > k0 ? (k1 - k0 + kKT - 1) / kKT : 0;

  // ---- issue the copies of one key tile (keys kt .. kt+63) into buffer buf
  auto load_tile = [&](int kt, int buf) {
    __nv_bfloat16* kd = ks + buf * kKT * D;
    __nv_bfloat16* vd = vs + buf * kKT * D;
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
    cp_async_commit();
  };

  if (n_tiles > 0) load_tile(k0, 0);

  // ---- Q rows r = j*B + i (query head h*g + j, block row i), zero rows past nr
  const int rows_pad = ((nr + 15) / 16) * 16;
  for (int e = tid; e < rows_pad * CH; e += nthr) {
    const int r = e / CH, c = e % CH;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nr) {
      const int j = r / p.B, i = r % p.B;
      v = *reinterpret_cast<const uint4*>(q + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + c * 8);
    }
    *reinterpret_cast<uint4*>(qs + swz<D>(r, c)) = v;
  }
  __syncthreads();

  const bool active = warp * 16 < nr;
  uint32_t qf[D / 16][4];
  if (active) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int mat = lane >> 3, r = lane & 7;
      ldsm_x4(qf[kk], qs + swz<D>(warp * 16 + r + 8 * (mat & 1), 2 * kk + (mat >> 1)));
    }
  }

  // fold 1/sqrt(d) and log2(e) into one factor: softmax runs in the exp2 domain
  const float sl2 = p.scale * 1.4426950408889634f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows gid and gid+8
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  for (int t = 0; t < n_tiles; ++t) {
    const int kt = k0 + t * kKT;
    if (t + 1 < n_tiles) {
      load_tile(kt + kKT, (t + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (active) {
      const __nv_bfloat16* kt_s = ks + (t & 1) * kKT * D;
      const __nv_bfloat16* vt_s = vs + (t & 1) * kKT * D;
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
      // mask keys past the split, scale, running max per row
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
    __syncthreads();
  }

  // ---- partial state of this split: unnormalised O, m (natural log units), l
  if (active) {
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, m);
      l1 += __shfl_xor_sync(0xffffffffu, l1, m);
    }
    const size_t pbase = ((size_t)(b * p.n_kv + h) * p.n_splits + s) * nr;
    const int r0 = warp * 16 + gid, r1 = r0 + 8;
    const float ln2 = 0.6931471805599453f;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int d = n * 8 + 2 * tig;
      if (r0 < nr) *reinterpret_cast<float2*>(p.part_o + (pbase + r0) * D + d) = make_float2(o[n][0], o[n][1]);
      if (r1 < nr) *reinterpret_cast<float2*>(p.part_o + (pbase + r1) * D + d) = make_float2(o[n][2], o[n][3]);
    }
    if (tig == 0) {
      if (r0 < nr) {
        p.part_m[pbase + r0] = m0 * ln2;
        p.part_l[pbase + r0] = l0;
      }
      if (r1 < nr) {
        p.part_m[pbase + r1] = m1 * ln2;
        p.part_l[pbase + r1] = l1;
      }
    }
  }
}

size_t attn_mma_smem_bytes(int d) { return (size_t)(128 + 4 * kKT) * d * 2; }

cudaError_t launch_attn_mma(const AttnParams& p, cudaStream_t st) {
  const int warps = (p.g * p.B + 15) / 16;
  const int threads = 32 * (warps < 4 ? 4 : warps);
  const size_t smem = attn_mma_smem_bytes(p.d);
  const dim3 grid(p.n_splits, p.n_kv, p.bs);
  if (p.d == 128) {
    static size_t set = 0;
    if (smem > set) {
      cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      set = smem;
    }
    attn_mma_kernel<128><<<grid, threads, smem, st>>>(p);
  } else {
    static size_t set = 0;
    if (smem > set) {
      cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      set = smem;
    }
    attn_mma_kernel<64><<<grid, threads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace dfl
