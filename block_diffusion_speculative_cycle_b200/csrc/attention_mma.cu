// Tensor-core block attention (fp16 operands, fp32 accumulate) for the bf16 drafter.
//
// One CTA per (split of the key range, KV head, request); the splits of one
// (request, KV head) form a thread-block cluster, or, for long contexts with few
// (request, KV head) pairs, write their partials to global memory for a merge
// kernel. The g*B block queries of the head group (g = n_q/n_kv query heads x B
// block rows, <= 128 rows) are split into 16-row slices; each slice has two warps
// (key groups), each taking half of every key tile, with the Q fragments read
// from shared memory for the mma.sync A operand. Keys
// stream through shared memory in tiles of 64 (a ring of 2-3 stages, cp.async 16-byte
// copies, XOR-swizzled rows so ldmatrix is conflict-free): context keys come
// from the request's cache pages, the B block keys from the block K/V rows
// (fp16, as the QKV projection writes them). A bf16 cache is converted to fp16
// in place once a tile lands, each thread converting the chunks it copied
// (exact for |v| < 65504); an fp16 cache is used as it is. The tensor-core
// operands are thus fp16: 11 significant bits for Q, the block K/V and the
// probabilities instead of bf16's 8.
// Per tile: S = Q·Kᵀ (m16n8k16), online softmax in fp32 (exp2 domain, quad
// shuffles), O += P·V with P re-packed from the S accumulators. The split's
// state (unnormalised O, running max m, sum l) is staged per row and each block
// of rows is bulk-copied into the receive buffer of the cluster CTA that owns
// those rows (distributed shared memory, counted on that CTA's mbarrier); each
// owner waits for exactly its rows, combines the splits (log-sum-exp weights,
// split order) and writes them as a pair of bf16 planes (hi, and lo = the
// rounding residue out_plane elements further on). The launcher instantiates
// KS = 2 only; the KS = 1 form (one warp per slice, Q held in registers) is kept
// in the template for reference and measurement.
#include "kernels.cuh"
#include "sm100.cuh"

namespace dfl {

namespace {

constexpr int kKT = 64;   // keys per tile

using sm100::smem_addr;
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return smem_addr(p); }
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
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Two bf16 (low half first) -> two fp16, through fp32 (a bf16 is the top half of an fp32).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
// Write v as hi = bf16(v) at dst and lo = bf16(v - hi) at dst + plane (two elements each).
__device__ __forceinline__ void store_split2(__nv_bfloat16* dst, size_t plane, float a, float b) {
  const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(hi);
  *reinterpret_cast<__nv_bfloat162*>(dst) = hi;
  *reinterpret_cast<__nv_bfloat162*>(dst + plane) = __floats2bfloat162_rn(a - hf.x, b - hf.y);
}

// Element offset of (row, 8-wide chunk) in a [rows][D] 16-bit tile with the
// 16-byte chunks of each row XOR-swizzled by row % 8.
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

}  // namespace

// Stages of the K/V ring: 3 for up to 64 query rows, 2 for 128. KS warp groups
// split every 64-key tile (KS = 2: group g takes keys 32g .. 32g+31), each with
// its own online-softmax state, merged in shared memory after the loop.
// With KS = 2 the Q fragments are re-read from shared memory for every tile
// instead of being held in registers, so the kernel fits 128 registers: two
// CTAs of 256 threads (<= 64 query rows) per SM, so that a 16-CTA cluster needs
// only 8 SMs of a GPC, or one CTA of 512 threads (128 query rows).
template <int D, int NST, int KS>
__global__ void __launch_bounds__(KS == 2 ? 512 : 256, KS == 2 ? 1 : 0) attn_cluster_kernel(const AttnParams p,
                                                                                            __nv_bfloat16* out) {
  constexpr bool kQReg = KS == 1;
  const size_t plane = p.out_plane;
  constexpr int CH = D / 8;          // 16-byte chunks per row
  constexpr int REC = D + 4;         // merge record: O (D floats), m, l, two pad words (16-byte multiple)
  constexpr int NT = kKT / 8 / KS;   // score n-tiles of 8 keys per warp group
  constexpr int KK = kKT / 16 / KS;  // P·V k-steps of 16 keys per warp group
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t recv_bar;
  const int nr = p.g * p.B;
  const int rows_pad = ((nr + 15) / 16) * 16;
  const int slices = rows_pad / 16;
  __half* qs = reinterpret_cast<__half*>(smem_raw);   // [rows_pad][D]
  __half* ring = qs + rows_pad * D;                    // NST x ([kKT][D] K, [kKT][D] V)
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int grp = warp / slices, slice = warp % slices;
  const int gid = lane >> 2, tig = lane & 3;
  const int q_dim = p.n_q * D, kv_dim = p.n_kv * D;
  const __half* q = reinterpret_cast<const __half*>(p.q);
  const __half* kb = reinterpret_cast<const __half*>(p.kblk);
  const __half* vb = reinterpret_cast<const __half*>(p.vblk);
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.kc);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.vc);
  // The context K/V were written by the injection kernels, which completed
  // before this kernel could be launched (each kernel of the chain waits for its
  // predecessor before it lets its successor start), and ctx_len / the page
  // table come from the caller. So the context tiles are fetched before the
  // wait; q and the block K/V come from the immediately preceding kernel.

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (tid == 0) flag_error(p.status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  const int T_all = P + p.B;
  // split s takes keys [base + s*kps, base + (s+1)*kps) (base: the 64-aligned start
  // of a sliding window, else 0); the last split also takes the rest (the block
  // keys of the longest requests run up to B past that); keys below ctx_lo are masked
  const int ctx_lo = attn_ctx_lo(P, p.window);
  const int k0 = min(T_all, attn_key_base(ctx_lo) + s * p.kps),
            k1 = s == p.n_splits - 1 ? T_all : min(T_all, k0 + p.kps);
  const int n_tiles = k1 > k0 ? (k1 - k0 + kKT - 1) / kKT : 0;

  const int S = p.n_splits;
  const bool gmerge = p.global_merge != 0;   // partials to global memory, merged by a second kernel
  if (gmerge && n_tiles == 0) return;         // a split past this request's keys: nothing to merge
  const int per = (nr + S - 1) / S;                       // merged rows owned by each split
  const int own_lo = min(nr, s * per), own_hi = min(nr, own_lo + per);
  if (S > 1 && !gmerge && tid == 0) {
    sm100::mbar_init(&recv_bar, 1);
    sm100::fence_mbar_init();
    sm100::mbar_arrive_expect_tx(&recv_bar, (uint32_t)(S * (own_hi - own_lo) * REC * 4));
  }

  // Tiles start at multiples of 64 keys (kps is a multiple of 64). When a tile
  // holds only context keys and the page size is a multiple of 64, its 64 keys
  // are one contiguous block of one page: resolve that page once.
  const bool page_tiles = (p.page_size % kKT) == 0;
  auto context_tile = [&](int kt) { return page_tiles && kt + kKT <= min(P, k1); };
  // Chunk e of a tile (row e / CH, 16-byte chunk e % CH) is always copied by
  // thread e % nthr, so after its own cp.async groups complete a thread can
  // convert the context chunks it copied without a barrier.
  auto tile_page = [&](int kt) {
    const int slot = kt / p.page_size;
    return slot < p.max_pages ? __ldg(p.page_table + (size_t)b * p.max_pages + slot) : -1;
  };
  // page: the tile's page when it is a context tile and the caller looked it up, else -2
  auto load_tile = [&](int kt, int stage, int page) {
    __half* kd = ring + stage * 2 * kKT * D;
    __half* vd = kd + kKT * D;
    if (context_tile(kt)) {
      if (page == -2) page = tile_page(kt);
      const bool ok = page >= 0 && page < p.num_pages;
      if (!ok && tid == 0) flag_error(p.status, ST_BAD_PAGE);
      const size_t base = ok ? (((size_t)page * p.n_kv + h) * p.page_size + kt % p.page_size) * D : 0;
      for (int e = tid; e < kKT * CH; e += nthr) {
        const int r = e / CH, c = e % CH;
        const size_t off = base + (size_t)r * D + c * 8;
        cp_async16(kd + swz<D>(r, c), ok ? kc + off : kc, ok ? 16 : 0);
        cp_async16(vd + swz<D>(r, c), ok ? vc + off : vc, ok ? 16 : 0);
      }
      return;
    }
    for (int e = tid; e < kKT * CH; e += nthr) {
      const int r = e / CH, c = e % CH, key = kt + r;
      const void* ksrc = kb;
      const void* vsrc = vb;
      int bytes = 0;
      if (key < k1 && key >= ctx_lo) {
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

  // the first NST tiles: pure-context ones now (their page ids fetched together),
  // the rest (and Q) after the wait
  int pg[NST];
#pragma unroll
  for (int i = 0; i < NST; ++i) pg[i] = i < n_tiles && context_tile(k0 + i * kKT) ? tile_page(k0 + i * kKT) : -2;
#pragma unroll
  for (int i = 0; i < NST; ++i)
    if (i < n_tiles && context_tile(k0 + i * kKT)) load_tile(k0 + i * kKT, i, pg[i]);
  cp_async_commit();
  grid_dep_wait();
  grid_dep_launch();
  // Q rows r = j*B + i: query head h*g + j, block row i
  for (int e = tid; e < rows_pad * CH; e += nthr) {
    const int r = e / CH, c = e % CH;
    const __half* src = q;
    int bytes = 0;
    if (r < nr) {
      const int j = r / p.B, i = r % p.B;
      src = q + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + c * 8;
      bytes = 16;
    }
    cp_async16(qs + swz<D>(r, c), src, bytes);
  }
#pragma unroll
  for (int i = 0; i < NST; ++i)
    if (i < n_tiles && !context_tile(k0 + i * kKT)) load_tile(k0 + i * kKT, i, -2);
  cp_async_commit();

  const bool active = slice * 16 < nr;
  uint32_t qf[D / 16][4];   // used when kQReg
  const float sl2 = p.scale * 1.4426950408889634f;   // softmax in the exp2 domain
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows gid, gid+8 of this slice
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  for (int t = 0; t < n_tiles; ++t) {
    // tiles < NST (and Q) landed with the two prologue groups; tile t >= NST with
    // the group committed NST iterations ago (one group per iteration)
    if (t == 0)
      cp_async_wait<0>();
    else
      cp_async_wait<NST - 1>();
    if (!p.cache_f16) {
      // context rows of this tile arrived as bf16: convert this thread's chunks
      const int kt = k0 + t * kKT;
      const int n_ctx = max(0, min(kKT, min(P, k1) - kt));
      uint4* kd = reinterpret_cast<uint4*>(ring + (t % NST) * 2 * kKT * D);
      uint4* vd = kd + kKT * D / 8;
      for (int e = tid; e < n_ctx * CH; e += nthr) {
        const int r = e / CH, c = e % CH;
        const int o16 = swz<D>(r, c) / 8;
        uint4 a = kd[o16], v = vd[o16];
        a.x = bf16x2_to_f16x2(a.x); a.y = bf16x2_to_f16x2(a.y); a.z = bf16x2_to_f16x2(a.z); a.w = bf16x2_to_f16x2(a.w);
        v.x = bf16x2_to_f16x2(v.x); v.y = bf16x2_to_f16x2(v.y); v.z = bf16x2_to_f16x2(v.z); v.w = bf16x2_to_f16x2(v.w);
        kd[o16] = a;
        vd[o16] = v;
      }
    }
    __syncthreads();
    if (active) {
      if (kQReg && t == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int mat = lane >> 3, r = lane & 7;
          ldsm_x4(qf[kk], qs + swz<D>(slice * 16 + r + 8 * (mat & 1), 2 * kk + (mat >> 1)));
        }
      }
      const int kt = k0 + t * kKT + grp * (kKT / KS);   // this group's first key
      const __half* kt_s = ring + (t % NST) * 2 * kKT * D + grp * (kKT / KS) * D;
      const __half* vt_s = ring + (t % NST) * 2 * kKT * D + kKT * D + grp * (kKT / KS) * D;
      float sc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int mat = lane >> 3, r = lane & 7;
        uint32_t qt[4];
        if constexpr (!kQReg) ldsm_x4(qt, qs + swz<D>(slice * 16 + r + 8 * (mat & 1), 2 * kk + (mat >> 1)));
#pragma unroll
        for (int n = 0; n < NT; n += 2) {
          const int kr = grp * (kKT / KS) + n * 8 + r + 8 * (mat >> 1);   // key row within the tile
          uint32_t bfr[4];
          ldsm_x4(bfr, ring + (t % NST) * 2 * kKT * D + swz<D>(kr, 2 * kk + (mat & 1)));
          if constexpr (kQReg) {
            mma_16816(sc[n], qf[kk], bfr[0], bfr[1]);
            mma_16816(sc[n + 1], qf[kk], bfr[2], bfr[3]);
          } else {
            mma_16816(sc[n], qt, bfr[0], bfr[1]);
            mma_16816(sc[n + 1], qt, bfr[2], bfr[3]);
          }
        }
      }
      (void)kt_s;
      float mx0 = m0, mx1 = m1;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int key = kt + n * 8 + 2 * tig;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const bool ok = key + c < k1 && key + c >= ctx_lo;
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
      // a group whose keys are all masked keeps its state (-inf max) untouched
      const float a0 = mx0 == -INFINITY ? 1.f : exp2f(m0 - mx0), a1 = mx1 == -INFINITY ? 1.f : exp2f(m1 - mx1);
      m0 = mx0;
      m1 = mx1;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pf[KK][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const float p00 = mx0 == -INFINITY ? 0.f : exp2f(sc[n][0] - m0);
        const float p01 = mx0 == -INFINITY ? 0.f : exp2f(sc[n][1] - m0);
        const float p10 = mx1 == -INFINITY ? 0.f : exp2f(sc[n][2] - m1);
        const float p11 = mx1 == -INFINITY ? 0.f : exp2f(sc[n][3] - m1);
        rs0 += p00 + p01;
        rs1 += p10 + p11;
        pf[n >> 1][(n & 1) * 2 + 0] = pack_f16(p00, p01);
        pf[n >> 1][(n & 1) * 2 + 1] = pack_f16(p10, p11);
      }
      l0 = l0 * a0 + rs0;
      l1 = l1 * a1 + rs1;
      // rescale the running O only when some row's max moved (after the first
      // tiles it rarely does); the test is warp-uniform
      if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= a0;
          o[n][1] *= a0;
          o[n][2] *= a1;
          o[n][3] *= a1;
        }
      }
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
        for (int n = 0; n < D / 8; n += 2) {
          const int mat = lane >> 3, r = lane & 7;
          const int kr = grp * (kKT / KS) + kk * 16 + r + 8 * (mat & 1);
          uint32_t bfr[4];
          ldsm_x4_t(bfr, ring + (t % NST) * 2 * kKT * D + kKT * D + swz<D>(kr, n + (mat >> 1)));
          mma_16816(o[n], pf[kk], bfr[0], bfr[1]);
          mma_16816(o[n + 1], pf[kk], bfr[2], bfr[3]);
        }
      }
      (void)vt_s;
    }
    __syncthreads();   // stage t % NST is free again
    if (t + NST < n_tiles) load_tile(k0 + (t + NST) * kKT, t % NST, -2);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();   // every copy has landed and every warp is done with Q and the ring
  // Past this barrier Q and the ring are dead; peers may write their merge records
  // into the tail of this CTA's shared memory once every CTA of the cluster arrives.
  if (S > 1 && !gmerge) sm100::cluster_arrive_release();

  if (active) {
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, m);
      l1 += __shfl_xor_sync(0xffffffffu, l1, m);
    }
  }
  const int r0 = slice * 16 + gid, r1 = r0 + 8;
  // [rows_pad][REC]: group 1's state for the group merge, then this split's records
  // (each group-0 thread rewrites the rows it read); [S][per][REC] received records
  float* grp_area = reinterpret_cast<float*>(smem_raw);
  float* stg = grp_area;
  float* rcv = grp_area + (size_t)rows_pad * REC;
  if (KS > 1) {
    // fold the second warp group's (O, m, l) into the first group's registers
    if (active && grp == 1) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float* rec = grp_area + (size_t)(half ? r1 : r0) * REC;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const int d = n * 8 + 2 * tig;
          *reinterpret_cast<float2*>(rec + d) = half ? make_float2(o[n][2], o[n][3]) : make_float2(o[n][0], o[n][1]);
        }
        if (tig == 0) {
          rec[D] = half ? m1 : m0;
          rec[D + 1] = half ? l1 : l0;
        }
      }
    }
    __syncthreads();
    if (active && grp == 0) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float* rec = grp_area + (size_t)(half ? r1 : r0) * REC;
        const float mo = rec[D], lo_ = rec[D + 1];
        float& mm = half ? m1 : m0;
        float& ll = half ? l1 : l0;
        const float M = fmaxf(mm, mo);
        const float wa = mm == -INFINITY ? 0.f : exp2f(mm - M), wb = mo == -INFINITY ? 0.f : exp2f(mo - M);
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const int d = n * 8 + 2 * tig;
          const float2 ov = *reinterpret_cast<const float2*>(rec + d);
          o[n][2 * half] = o[n][2 * half] * wa + ov.x * wb;
          o[n][2 * half + 1] = o[n][2 * half + 1] * wa + ov.y * wb;
        }
        ll = ll * wa + lo_ * wb;
        mm = M;
      }
    }
    __syncwarp();   // every lane has read its rows' m and l before they are overwritten below
  }
  const bool writer = active && grp == 0;
  if (gmerge) {
    // this split's unnormalised O, max and sum per row (exp2 domain) for the merge kernel
    const size_t pbase = ((size_t)(b * p.n_kv + h) * S + s) * nr;
    if (writer) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = half ? r1 : r0;
        if (r < nr) {
          float* po = p.part_o + (pbase + r) * D;
#pragma unroll
          for (int n = 0; n < D / 8; ++n) {
            const int d = n * 8 + 2 * tig;
            *reinterpret_cast<float2*>(po + d) = half ? make_float2(o[n][2], o[n][3]) : make_float2(o[n][0], o[n][1]);
          }
          if (tig == 0) {
            p.part_m[pbase + r] = half ? m1 : m0;
            p.part_l[pbase + r] = half ? l1 : l0;
          }
        }
      }
    }
    return;
  }
  if (S == 1) {
    // the whole key range is here: normalise and write
    if (writer) {
      const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        const int d = n * 8 + 2 * tig;
        if (r0 < nr) {
          const int j = r0 / p.B, i = r0 % p.B;
          store_split2(out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + d, plane, o[n][0] * i0,
                       o[n][1] * i0);
        }
        if (r1 < nr) {
          const int j = r1 / p.B, i = r1 % p.B;
          store_split2(out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D + d, plane, o[n][2] * i1,
                       o[n][3] * i1);
        }
      }
    }
    return;
  }

  // ---- cluster merge: stage this split's (O, m, l) records, bulk-copy each
  // owner's block of rows into its receive buffer (counted on its barrier), then
  // combine the rows this split owns over all splits, in split order.
  if (writer) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = half ? r1 : r0;
      if (r < nr) {
        float* rec = stg + (size_t)r * REC;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const int d = n * 8 + 2 * tig;
          *reinterpret_cast<float2*>(rec + d) = half ? make_float2(o[n][2], o[n][3]) : make_float2(o[n][0], o[n][1]);
        }
        if (tig == 0) {
          rec[D] = half ? m1 : m0;
          rec[D + 1] = half ? l1 : l0;
        }
      }
    }
  }
  sm100::fence_proxy_async_smem();
  __syncthreads();
  sm100::cluster_wait_acquire();   // every CTA is past its loop and its receive barrier is set
  if (tid == 0) {
    const uint32_t rcv_s = smem_u32(rcv), bar_s = smem_u32(&recv_bar), stg_s = smem_u32(stg);
    for (int k = 0; k < S; ++k) {
      const int lo = min(nr, k * per), hi = min(nr, lo + per);
      if (hi > lo)
        sm100::bulk_copy_s2s(sm100::mapa_shared(rcv_s + (uint32_t)(s * per * REC * 4), (uint32_t)k),
                             stg_s + (uint32_t)(lo * REC * 4), (uint32_t)((hi - lo) * REC * 4),
                             sm100::mapa_shared(bar_s, (uint32_t)k));
    }
    sm100::bulk_commit();
  }
  const bool got = sm100::mbar_wait(&recv_bar, 0, p.status);
  const int nwarps = nthr >> 5;
  for (int r = own_lo + warp; got && r < own_hi; r += nwarps) {
    const int rl = r - own_lo;
    const float ms = lane < S ? rcv[((size_t)lane * per + rl) * REC + D] : -INFINITY;
    const float ls = lane < S ? rcv[((size_t)lane * per + rl) * REC + D + 1] : 0.f;
    float M = ms;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    const float w = (lane < S && ms != -INFINITY) ? exp2f(ms - M) : 0.f;
    float L = ls * w;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) L += __shfl_xor_sync(0xffffffffu, L, m);
    const float invL = 1.f / L;
    float acc[D / 32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
    for (int k = 0; k < S; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float* src = rcv + ((size_t)k * per + rl) * REC;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(wk, src[lane + 32 * c], acc[c]);
    }
    const int j = r / p.B, i = r % p.B;
    __nv_bfloat16* dst = out + (size_t)(b * p.B + i) * q_dim + (h * p.g + j) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const float v = acc[c] * invL;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      dst[lane + 32 * c] = hi;
      dst[lane + 32 * c + plane] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
  if (tid == 0) sm100::bulk_wait_read_all();   // the staging has been read by every outgoing copy
}

static size_t attn_cluster_smem(int d, int nr, int rows_pad, int nst, int ks, int splits, bool gmerge) {
  const size_t loads = ((size_t)rows_pad + (size_t)nst * 2 * kKT) * d * 2;
  const size_t per = (size_t)(nr + splits - 1) / splits;
  const size_t rec = (size_t)(d + 4) * 4;
  const bool cl = splits > 1 && !gmerge;
  const size_t merge = (ks > 1 || cl ? (size_t)rows_pad * rec : 0) + (cl ? splits * per * rec : 0);
  return loads > merge ? loads : merge;
}

// Global merge (many splits): one CTA per (block row, query head). Its four warps
// take the splits that hold keys in turn (split s to warp s % 4), each lane a
// contiguous run of D/32 output columns, so every warp has its loads in flight
// together; the warps' sums meet in shared memory. Log-sum-exp weights in the
// exp2 domain; the row is written as bf16 hi/lo planes.
template <int D>
__global__ void __launch_bounds__(128) attn_gmerge_kernel(const AttnParams p, __nv_bfloat16* out) {
  constexpr int DPL = D / 32;   // columns per lane: 4 (D = 128) or 2 (D = 64)
  __shared__ float red_m[4], red_l[4];
  __shared__ __align__(16) float red_o[4][D];
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_row = blockIdx.x / p.n_q, j = blockIdx.x % p.n_q;
  const int b = m_row / p.B, i = m_row % p.B;
  const int h = j / p.g, jj = j % p.g;
  const int nr = p.g * p.B, r = jj * p.B + i;
  int P = p.ctx_len[b];
  P = P < 0 ? 0 : (P > p.max_ctx ? p.max_ctx : P);
  const int kps = attn_kps(p);
  const int used = min(p.n_splits, (P + p.B - attn_key_base(attn_ctx_lo(P, p.window)) + kps - 1) / kps);
  const size_t base = (size_t)(b * p.n_kv + h) * p.n_splits * nr + r;
  // the row's maximum over the splits
  float M = -INFINITY;
  for (int s = threadIdx.x; s < used; s += 128) M = fmaxf(M, __ldcg(p.part_m + base + (size_t)s * nr));
  M = warp_max(M);
  if (lane == 0) red_m[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
  // this warp's splits: sum of 2^(m_s - M) * (l_s, o_s)
  float acc[DPL], L = 0.f;
#pragma unroll
  for (int c = 0; c < DPL; ++c) acc[c] = 0.f;
#pragma unroll 4
  for (int s = warp; s < used; s += 4) {
    const size_t idx = base + (size_t)s * nr;
    const float ms = __ldcg(p.part_m + idx);
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
    L = fmaf(w, __ldcg(p.part_l + idx), L);
    const float* o = p.part_o + idx * D + lane * DPL;
    if constexpr (DPL == 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(o));
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
      acc[2] = fmaf(w, v.z, acc[2]);
      acc[3] = fmaf(w, v.w, acc[3]);
    } else {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(o));
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
    }
  }
  if (lane == 0) red_l[warp] = L;
#pragma unroll
  for (int c = 0; c < DPL; ++c) red_o[warp][lane * DPL + c] = acc[c];
  __syncthreads();
  if (threadIdx.x < D) {
    const int col = threadIdx.x;
    const float Lt = (red_l[0] + red_l[1]) + (red_l[2] + red_l[3]);
    const float v = ((red_o[0][col] + red_o[1][col]) + (red_o[2][col] + red_o[3][col])) / Lt;
    __nv_bfloat16* dst = out + (size_t)m_row * p.n_q * D + j * D + col;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    dst[0] = hi;
    dst[p.out_plane] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

cudaError_t launch_attn_gmerge(const AttnParams& p, void* out, cudaStream_t st, bool pdl) {
  const int rows = p.bs * p.B * p.n_q;
  if (p.d == 128)
    return launch_kernel(attn_gmerge_kernel<128>, dim3(rows), dim3(128), 0, st, pdl, p, (__nv_bfloat16*)out);
  if (p.d == 64)
    return launch_kernel(attn_gmerge_kernel<64>, dim3(rows), dim3(128), 0, st, pdl, p, (__nv_bfloat16*)out);
  return cudaErrorInvalidValue;
}

template <int D, int NST, int KS>
static cudaError_t launch_cluster_t(const AttnParams& p, void* out, cudaStream_t st, bool pdl) {
  const int nr = p.g * p.B;
  const int rows_pad = ((nr + 15) / 16) * 16;
  const int threads = 32 * KS * (rows_pad / 16);
  const bool gmerge = p.global_merge != 0;
  const size_t smem = attn_cluster_smem(D, nr, rows_pad, NST, KS, p.n_splits, gmerge);
  static size_t set = 0;
  if (smem > set) {
    cudaError_t e = cudaFuncSetAttribute(attn_cluster_kernel<D, NST, KS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_cluster_kernel<D, NST, KS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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
  cfg.numAttrs = p.n_splits > 1 && !gmerge ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_cluster_kernel<D, NST, KS>, p, (__nv_bfloat16*)out);
  if (e != cudaSuccess || !gmerge) return e;
  return launch_attn_gmerge(p, out, st, pdl);
}

cudaError_t launch_attn_cluster(const AttnParams& p, void* out, cudaStream_t st, bool pdl) {
  if (p.n_splits < 1 || (!p.global_merge && p.n_splits > kMaxAttnCluster) || p.kps % kKT) return cudaErrorInvalidValue;
  // Two key groups per CTA (every launch): two warps per 16 query rows, each
  // taking half of every key tile; a two-stage ring (three at d = 64 and <= 64
  // rows when a CTA streams more than two tiles: two CTAs per SM still fit).
  if (p.ks != 2) return cudaErrorInvalidValue;
  if (p.d == 128) return launch_cluster_t<128, 2, 2>(p, out, st, pdl);
  const bool three = p.g * p.B <= 64 && p.kps / kKT > 2;
  return three ? launch_cluster_t<64, 3, 2>(p, out, st, pdl) : launch_cluster_t<64, 2, 2>(p, out, st, pdl);
}

}  // namespace dfl
