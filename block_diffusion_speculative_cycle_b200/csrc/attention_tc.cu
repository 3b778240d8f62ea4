// Block attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA) for
// the bf16 drafter with an fp16 KV cache.
//
// What it computes ("DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩" §6:
// in-block attention is non-causal; "DFlash – 플래시 추측적 디코딩을 위한 블록 확산"
// §2.2: the block attends to the context K/V injected into the drafter cache):
// for request b and KV head h, every one of the g*B query rows (g query heads of
// the group x B block rows) attends, with no mask, to the request's P context
// keys and all B block keys: o = softmax(q·Kᵀ/√d)·V.
//
// One CTA per (split of the key range, KV head, request). The key range of a
// request is the P context keys followed by the B block keys; split s takes keys
// [s*kps, (s+1)*kps) of it (the last split everything left). Context keys come
// from the cache pages (64-key tiles, one page and head each), block keys from
// the block k/v rows the QKV projection wrote; a tile never mixes the two.
//
// Warp roles (192 threads):
//   warp 0     TMA producer (one lane): Q once, then K/V tiles into a ring of stages
//   warp 1     TMEM owner + MMA issuer (one lane):
//                S_t = Q·K_tᵀ   M = 128 query rows (zero-padded), N = 64 keys, K = d
//                O  += P_t·V_t  M = 128, N = d, K = 64 keys (V read MN-major)
//              S is double-buffered in TMEM (2 x 64 columns), O has d columns.
//   warps 2-5  softmax: each thread owns one query row (= one TMEM lane); reads
//              its S row with tcgen05.ld, keeps a running max and sum in the
//              exp2 domain, writes P (fp16) to shared memory in the MMA's
//              swizzled K-major layout. The running max is raised lazily: only
//              when a row's max grows by more than 2^8 is O rescaled in TMEM
//              (tcgen05.ld / st) and the sum with it, so P stays <= 2^8 in fp16.
// After the last tile the rows' (O, m, l) are merged across the splits of the
// (request, head): through distributed shared memory inside a cluster, or, for
// many splits, through global memory and a second kernel. Every wait is bounded;
// on a timeout the CTA flags ST_TIMEOUT, stops, lets its copies and MMAs finish,
// still takes part in every cluster barrier, frees TMEM and returns.
#include "kernels.cuh"
#include "sm100.cuh"

namespace dfl {

using namespace sm100;

namespace {

constexpr int kKT = 64;           // keys per tile
constexpr int kThreads = 192;
constexpr int kRows = 128;        // MMA M (query rows, zero-padded)
constexpr int kTmemCols = 256;    // S: 2 x 64 columns, O: d columns from column 128
constexpr int kOCol = 128;
constexpr float kLazyLog2 = 8.f;  // raise the running max only past 2^8

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnTcParams tp,
                                                              __nv_bfloat16* out) {
  constexpr int HALVES = D / 64;                 // 64-element (128-byte) column blocks of a row
  constexpr int QH = kRows * 128;                // one column block of Q (16 KB)
  constexpr int KH = kKT * 128;                  // one column block of a K or V tile (8 KB)
  constexpr int STAGE = 2 * HALVES * KH;         // K + V of one tile
  constexpr int PB = kRows * kKT * 2;            // one P buffer (16 KB)
  constexpr int REC = D + 4;                     // merge record: O, m, l, 2 pad words
  const AttnParams& p = tp.a;
  const int NST = tp.stages;

  extern __shared__ uint8_t dsm_raw[];
  __shared__ uint64_t q_full, fin_bar, recv_bar;
  __shared__ uint64_t pv_done[2];   // pv_done[u & 1]: the P·V of tile u has completed
  __shared__ uint64_t kv_full[kMaxAttnTcStages], kv_empty[kMaxAttnTcStages];
  __shared__ uint64_t s_full[2], s_free[2], p_full[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int s_abort;

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = base;
  uint8_t* ring = qs + HALVES * QH;
  uint8_t* pbuf = ring + (size_t)NST * STAGE;

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nr = p.g * p.B;
  int* status = p.status;

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (threadIdx.x == 0) flag_error(status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  // this split's keys: [k0, k1) of the sequence (P context keys, then B block keys)
  const int S = p.n_splits;
  const int T_all = P + p.B;
  const int k0 = min(T_all, s * p.kps);
  const int k1 = s == S - 1 ? T_all : min(T_all, k0 + p.kps);
  const int cx1 = min(k1, P);                               // context part [k0, cx1)
  const int n_ctx = cx1 > k0 ? (cx1 - k0 + kKT - 1) / kKT : 0;
  const int bk0 = max(k0, P) - P, bk1 = k1 - P;             // block rows [bk0, bk1)
  const int n_blk = bk1 > bk0 ? (bk1 - bk0 + kKT - 1) / kKT : 0;
  const int n_tiles = n_ctx + n_blk;
  auto tile_valid = [&](int t) {
    return t < n_ctx ? min(kKT, cx1 - (k0 + t * kKT)) : min(kKT, bk1 - (bk0 + (t - n_ctx) * kKT));
  };

  const bool gmerge = p.global_merge != 0;
  if (gmerge && n_tiles == 0) return;   // nothing of this request here: the merge kernel skips the split
  const bool cluster = S > 1 && !gmerge;
  const int per = (nr + S - 1) / S;     // merged rows owned by each split (cluster merge)
  const int own_lo = min(nr, s * per), own_hi = min(nr, own_lo + per);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&fin_bar, 1);
    mbar_init(&recv_bar, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
    }
    s_abort = 0;
    fence_mbar_init();
    if (cluster) mbar_arrive_expect_tx(&recv_bar, (uint32_t)(S * (own_hi - own_lo) * REC * 4));
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tp.kcmap);
    prefetch_tmap(&tp.vcmap);
    prefetch_tmap(&tp.qmap);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // rows nr..127 of Q are padding: zero them (the MMA reads 128 rows)
  {
    const int pad_chunks = (kRows - nr) * 8;   // 16-byte chunks per column block
    for (int e = threadIdx.x; e < pad_chunks * HALVES; e += kThreads) {
      const int hh = e / pad_chunks, c = e % pad_chunks;
      *reinterpret_cast<uint4*>(qs + hh * QH + nr * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // softmax threads' results, kept in registers across the block barrier below
  float o[D];
  float m_used = -INFINITY, l = 0.f;
  const int row = (warp & 3) * 32 + lane;   // softmax warps: query row (= TMEM lane) of this thread

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      const uint64_t pol = policy_evict_first();
      auto issue = [&](int t, int st) {
        uint8_t* kd = ring + (size_t)st * STAGE;
        uint8_t* vd = kd + HALVES * KH;
        mbar_arrive_expect_tx(&kv_full[st], (uint32_t)STAGE);
        if (t < n_ctx) {
          const int kt = k0 + t * kKT;
          const int slot = kt / p.page_size;
          int page = slot < p.max_pages ? __ldg(p.page_table + (size_t)b * p.max_pages + slot) : -1;
          if (page < 0 || page >= p.num_pages) {
            flag_error(status, ST_BAD_PAGE);
            page = 0;   // read a valid page instead; the result is flagged as wrong
          }
          const int row = (page * p.n_kv + h) * p.page_size + kt % p.page_size;
#pragma unroll
          for (int hh = 0; hh < HALVES; ++hh) {
            tma_load_2d(kd + hh * KH, &tp.kcmap, &kv_full[st], hh * 64, row, pol);
            tma_load_2d(vd + hh * KH, &tp.vcmap, &kv_full[st], hh * 64, row, pol);
          }
        } else {
          const int r0 = bk0 + (t - n_ctx) * kKT;
#pragma unroll
          for (int hh = 0; hh < HALVES; ++hh) {
            tma_load_3d(kd + hh * KH, &tp.kbmap, &kv_full[st], h * D + hh * 64, r0, b, pol);
            tma_load_3d(vd + hh * KH, &tp.vbmap, &kv_full[st], h * D + hh * 64, r0, b, pol);
          }
        }
      };
      const int pre = min(n_tiles, NST);
      // Context tiles were written by earlier kernels of the stream, all complete
      // by now (every kernel waits for its predecessor before letting its
      // successor start): fetch them before waiting on the previous kernel.
      for (int t = 0; t < pre; ++t)
        if (t < n_ctx) issue(t, t);
      grid_dep_wait();
      mbar_arrive_expect_tx(&q_full, (uint32_t)(HALVES * nr * 128));
#pragma unroll
      for (int hh = 0; hh < HALVES; ++hh)
        tma_load_3d(qs + hh * QH, &tp.qmap, &q_full, hh * 64, h * p.g, b * p.B, pol);
      for (int t = 0; t < pre; ++t)
        if (t >= n_ctx) issue(t, t);
      int issued = pre;
      for (int t = pre; t < n_tiles; ++t) {
        const int st = t % NST;
        if (s_abort || !mbar_wait(&kv_empty[st], ((t / NST) & 1) ^ 1, status)) {
          s_abort = 1;
          break;
        }
        issue(t, st);
        ++issued;
      }
      grid_dep_launch();
      // let every copy this CTA issued land before the CTA can exit
      mbar_wait(&q_full, 0, status);
      for (int t = max(0, issued - NST); t < issued; ++t) mbar_wait(&kv_full[t % NST], (t / NST) & 1, status);
    } else if (lane == 0) {
      grid_dep_wait();
      grid_dep_launch();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t id_s = idesc_f16_f32(kRows, kKT, 0);
      const uint32_t id_o = idesc_f16_f32(kRows, D, 1);
      auto pv = [&](int u) -> bool {
        if (s_abort || !mbar_wait(&p_full[u & 1], (u >> 1) & 1, status)) return false;
        tc_fence_after();
        const uint32_t vd = smem_addr(ring + (size_t)(u % NST) * STAGE + HALVES * KH);
        const uint32_t pb = smem_addr(pbuf + (u & 1) * PB);
        const uint64_t ad = desc_kmajor_sw128(pb);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)   // 16 keys per MMA: +32 B in P's rows, +2 KB (16 rows) in V
          mma_bf16(tmem + kOCol, ad + (uint64_t)(2 * kk), desc_mnmajor_sw128(vd + kk * 2048, KH), id_o,
                   (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&pv_done[u & 1]);
        mma_commit(&kv_empty[u % NST]);
        return true;
      };
      bool ok = mbar_wait(&q_full, 0, status);
      int t = 0;
      for (; ok && t < n_tiles; ++t) {
        const int st = t % NST;
        ok = !s_abort && mbar_wait(&kv_full[st], (t / NST) & 1, status);
        if (ok && t >= 2) ok = !s_abort && mbar_wait(&s_free[t & 1], ((t >> 1) - 1) & 1, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kd = smem_addr(ring + (size_t)st * STAGE);
        const uint32_t qa = smem_addr(qs);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // K = d in steps of 16: +32 B inside a 128-byte block
          const int hh = kk >> 2, sub = kk & 3;
          mma_bf16(tmem + (uint32_t)((t & 1) * kKT), desc_kmajor_sw128(qa + hh * QH) + (uint64_t)(2 * sub),
                   desc_kmajor_sw128(kd + hh * KH) + (uint64_t)(2 * sub), id_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[t & 1]);
        if (t >= 1 && !(ok = pv(t - 1))) break;
      }
      if (ok) ok = pv(n_tiles - 1);
      if (!ok) s_abort = 1;
      // every MMA issued has completed before TMEM can be freed
      mma_commit(&fin_bar);
      mbar_wait(&fin_bar, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int qd = warp & 3;                       // TMEM lane quarter this warp may access
    const int tid = threadIdx.x - 64;              // 0..127
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    const float sl2 = p.scale * 1.4426950408889634f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      ok = !s_abort && mbar_wait(&s_full[t & 1], (t >> 1) & 1, status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; s_abort = 1; break; }
      tc_fence_after();
      uint32_t sr[kKT];
      tmem_ld32_nowait(lane_addr + (uint32_t)((t & 1) * kKT), sr);
      tmem_ld32_nowait(lane_addr + (uint32_t)((t & 1) * kKT + 32), sr + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[t & 1]);
      const int valid = tile_valid(t);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKT; ++c) {
        const float v = c < valid ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
        sr[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      // the P buffer of this tile was last read by the P·V of tile t-2 (one
      // barrier per P buffer: its phases are that buffer's P·V launches, so at most
      // one of them can complete past the one waited for)
      if (t >= 2) ok = mbar_wait(&pv_done[t & 1], ((t - 2) >> 1) & 1, status);
      float alpha = 1.f;
      bool resc = false;
      if (m_used == -INFINITY) {
        m_used = mx;   // first keys of this row: nothing accumulated yet
      } else if (mx > m_used + kLazyLog2) {
        alpha = exp2f(m_used - mx);
        m_used = mx;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O holds tiles < t: wait for the P·V of tile t-1, then rescale this warp's rows
        if (ok) ok = mbar_wait(&pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, status);
        if (__all_sync(0xffffffffu, ok)) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld32_nowait(lane_addr + (uint32_t)(kOCol + c0), r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(lane_addr + (uint32_t)(kOCol + c0), r);
          }
          tmem_wait_st();
        }
        l *= alpha;
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; s_abort = 1; break; }
      // P row (fp16, <= 2^8) into the K-major, 128-byte-swizzled P buffer
      float sum = 0.f;
      uint8_t* prow = pbuf + (t & 1) * PB + row * 128;
#pragma unroll
      for (int j = 0; j < kKT / 8; ++j) {
        float e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          e[i] = m_used == -INFINITY ? 0.f : exp2f(__uint_as_float(sr[8 * j + i]) - m_used);
          sum += e[i];
        }
        *reinterpret_cast<uint4*>(prow + ((j ^ (row & 7)) << 4)) =
            make_uint4(pack_f16x2(e[0], e[1]), pack_f16x2(e[2], e[3]), pack_f16x2(e[4], e[5]),
                       pack_f16x2(e[6], e[7]));
      }
      l += sum;
      // a partial tile: V rows past the valid keys may hold anything (even NaN,
      // which a zero probability would not cancel); zero them
      if (valid < kKT) {
        uint8_t* vd = ring + (size_t)(t % NST) * STAGE + HALVES * KH;
        const int n = (kKT - valid) * 8;
        for (int e = tid; e < n * HALVES; e += 128) {
          const int hh = e / n, c = e % n;
          *reinterpret_cast<uint4*>(vd + hh * KH + valid * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[t & 1]);
    }
    // final O row
    bool have = ok && n_tiles > 0;
    if (have) have = mbar_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, status);
    if (__all_sync(0xffffffffu, have)) {
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32_nowait(lane_addr + (uint32_t)(kOCol + c0), r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c0 + i] = __uint_as_float(r[i]);
      }
    } else {
      if (n_tiles > 0) s_abort = 1;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = 0.f;
      m_used = -INFINITY;
      l = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();   // ring, Q and TMEM are dead for every role
  if (cluster) cluster_arrive_release();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (warp >= 2) {
    const int i_blk = row / p.g, j_head = row % p.g;   // TMA wrote Q rows in (block row, head) order
    if (gmerge) {
      if (row < nr) {
        const size_t pr = ((size_t)(b * p.n_kv + h) * S + s) * nr + (size_t)j_head * p.B + i_blk;
        float* po = p.part_o + pr * D;
#pragma unroll
        for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(po + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        p.part_m[pr] = m_used;
        p.part_l[pr] = l;
      }
    } else if (!cluster) {
      if (row < nr) {
        const float inv = 1.f / l;
        __nv_bfloat16* dst = out + (size_t)(b * p.B + i_blk) * (p.n_q * D) + (size_t)(h * p.g + j_head) * D;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a = o[c + 2 * k] * inv, bb = o[c + 2 * k + 1] * inv;
            const __nv_bfloat162 hv = __floats2bfloat162_rn(a, bb);
            const float2 hf = __bfloat1622float2(hv);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(a - hf.x, bb - hf.y);
            hi[k] = *reinterpret_cast<const uint32_t*>(&hv);
            lo[k] = *reinterpret_cast<const uint32_t*>(&lv);
          }
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(dst + c + p.out_plane) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    } else if (row < nr) {
      float* rec = reinterpret_cast<float*>(base) + (size_t)row * REC;
#pragma unroll
      for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(rec + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      rec[D] = m_used;
      rec[D + 1] = l;
    }
  }
  if (!cluster) return;

  // ---- cluster merge: each owner gets every split's records of its rows
  float* stg = reinterpret_cast<float*>(base);
  float* rcv = stg + (size_t)kRows * REC;
  fence_proxy_async_smem();
  __syncthreads();
  cluster_wait_acquire();   // every CTA is past its loop and its receive barrier is set
  if (threadIdx.x == 0) {
    const uint32_t rcv_s = smem_addr(rcv), bar_s = smem_addr(&recv_bar), stg_s = smem_addr(stg);
    for (int k = 0; k < S; ++k) {
      const int lo = min(nr, k * per), hi = min(nr, lo + per);
      if (hi > lo)
        bulk_copy_s2s(mapa_shared(rcv_s + (uint32_t)(s * per * REC * 4), (uint32_t)k),
                      stg_s + (uint32_t)(lo * REC * 4), (uint32_t)((hi - lo) * REC * 4), mapa_shared(bar_s, (uint32_t)k));
    }
    bulk_commit();
  }
  const bool got = mbar_wait(&recv_bar, 0, status);
  constexpr int nwarps = kThreads / 32;
  for (int r = own_lo + warp; got && r < own_hi; r += nwarps) {
    const int rl = r - own_lo;
    const float ms = lane < S ? rcv[((size_t)lane * per + rl) * REC + D] : -INFINITY;
    const float ls = lane < S ? rcv[((size_t)lane * per + rl) * REC + D + 1] : 0.f;
    const float M = warp_max(ms);
    const float w = (lane < S && ms != -INFINITY) ? exp2f(ms - M) : 0.f;
    const float invL = 1.f / warp_sum(ls * w);
    float acc[D / 32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
    for (int k = 0; k < S; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float* src = rcv + ((size_t)k * per + rl) * REC;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(wk, src[lane + 32 * c], acc[c]);
    }
    const int i = r / p.g, j = r % p.g;
    __nv_bfloat16* dst = out + (size_t)(b * p.B + i) * (p.n_q * D) + (size_t)(h * p.g + j) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const float v = acc[c] * invL;
      const __nv_bfloat16 hv = __float2bfloat16_rn(v);
      dst[lane + 32 * c] = hv;
      dst[lane + 32 * c + p.out_plane] = __float2bfloat16_rn(v - __bfloat162float(hv));
    }
  }
  if (threadIdx.x == 0) bulk_wait_read_all();   // the staging has been read by every outgoing copy
}

size_t attn_tc_smem_bytes(int d, int stages, int splits, bool gmerge, int nr) {
  const int halves = d / 64;
  const size_t loads = (size_t)halves * kRows * 128 + (size_t)stages * 2 * halves * kKT * 128 + 2 * (size_t)kRows * kKT * 2;
  const size_t rec = (size_t)(d + 4) * 4;
  const size_t per = (size_t)(nr + splits - 1) / splits;
  const size_t merge = splits > 1 && !gmerge ? ((size_t)kRows + (size_t)splits * per) * rec : 0;
  return (loads > merge ? loads : merge) + 1024;
}

template <int D>
static cudaError_t launch_tc_t(const AttnTcParams& tp, void* out, cudaStream_t st, bool pdl) {
  const AttnParams& p = tp.a;
  const bool gmerge = p.global_merge != 0;
  const size_t smem = attn_tc_smem_bytes(D, tp.stages, p.n_splits, gmerge, p.g * p.B);
  static size_t set = 0;
  if (smem > set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    set = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, p.n_kv, p.bs);
  cfg.blockDim = dim3(kThreads);
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
  void* args[] = {const_cast<AttnTcParams*>(&tp), &out};
  cudaError_t e = cudaLaunchKernelExC(&cfg, (const void*)attn_tc_kernel<D>, args);
  if (e != cudaSuccess || !gmerge) return e;
  return launch_attn_gmerge(p, out, st, pdl);
}

cudaError_t launch_attn_tc(const AttnTcParams& tp, void* out, cudaStream_t st, bool pdl) {
  const AttnParams& p = tp.a;
  if (p.n_splits < 1 || (!p.global_merge && p.n_splits > kMaxAttnCluster) || p.kps % kKT || p.page_size % kKT)
    return cudaErrorInvalidValue;
  if (tp.stages < 2 || tp.stages > kMaxAttnTcStages || p.g * p.B > kRows) return cudaErrorInvalidValue;
  if (p.d == 128) return launch_tc_t<128>(tp, out, st, pdl);
  if (p.d == 64) return launch_tc_t<64>(tp, out, st, pdl);
  return cudaErrorInvalidValue;
}

// Clusters of n CTAs of this kernel's shape that can be resident at once (0: none fit).
int attn_tc_max_clusters(int d, int stages, int n, bool gmerge, int nr) {
  const size_t smem = attn_tc_smem_bytes(d, stages, n, gmerge, nr);
  const void* k = d == 128 ? (const void*)attn_tc_kernel<128> : (const void*)attn_tc_kernel<64>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 0;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n, 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)n;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int num = 0;
  if (cudaOccupancyMaxActiveClusters(&num, k, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return num;
}

}  // namespace dfl
