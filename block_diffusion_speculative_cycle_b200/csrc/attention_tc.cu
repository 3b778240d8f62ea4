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
// Warp roles:
//   warp 0     TMA producer (one lane): Q once, then K/V tiles into a ring of stages
//   warp 1     TMEM owner + MMA issuer (one lane):
//                S_t = Q·K_tᵀ   M = 128 query rows (padded), N = 64 keys, K = d
//                O  += P_t·V_t  M = 128, N = d, K = 64 keys (V read MN-major)
//              S (then P over it, as fp16 pairs) sits in a ring of 2 or 4 TMEM
//              buffers of 64 columns; O has d columns after them.
//   warps 2..  softmax, WPQ warps per TMEM lane quarter (a warp may only read the
//              32 lanes of its quarter): each thread owns one query row (= one
//              TMEM lane) and 64/WPQ of the tile's key columns; it reads them with
//              tcgen05.ld, the row's maximum is combined across the WPQ threads
//              of the row through shared memory, and it keeps a running max and
//              sum in the exp2 domain and writes its part of P (fp16 pairs) back
//              over the tile's S in TMEM (tcgen05.st), where the P·V MMA reads its
//              A operand. The running max is raised lazily: only when a row's max
//              grows by more than 2^8 is O rescaled in TMEM (tcgen05.ld / st) and
//              the sum with it, so P stays <= 2^8 in fp16.
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
constexpr int kRows = 128;        // MMA M (query rows; rows past g*B are padding)
constexpr float kLazyLog2 = 8.f;  // raise the running max only past 2^8

// S/P buffers in TMEM (64 columns each; S may run this many tiles ahead of the
// P·V) and the TMEM columns a CTA takes: compact 2 buffers + O in 256 columns (two
// CTAs per SM), full 4 buffers + O in 512.
__host__ __device__ constexpr int tc_nsb(bool compact) { return compact ? 2 : 4; }
__host__ __device__ constexpr int tc_tmem_cols(bool compact) { return compact ? 256 : 512; }
// Softmax warps per TMEM lane quarter: 2 in the compact form (two CTAs per SM), 4 otherwise.
__host__ __device__ constexpr int tc_wpq(bool compact) { return compact ? 2 : 4; }
__host__ __device__ constexpr int tc_threads(bool compact) { return 64 + 128 * tc_wpq(compact); }

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// 2^x on the special-function unit (relative error ~2^-22, far below the fp16
// rounding the probabilities get); 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace

__device__ __forceinline__ int p_rows_of(const AttnTcParams& tp) { return tp.a.g * tp.a.B; }

// COMPACT: two CTAs share an SM (a two-stage ring, two S/P buffers, 8 softmax
// warps, 256 TMEM columns, at most about 100 KB). With at most 64 query rows Q
// takes 64 rows per column block (the MMA's rows 64..127 then read whatever
// follows and give TMEM lanes 64..127, which nothing reads); otherwise, and in the
// full form (one CTA per SM, `stages` stages, 4 S/P buffers, 16 softmax warps),
// Q is zero-padded to 128 rows.
// The S buffer of tile t is reused for tile t + NSB once the P·V of tile t (which
// reads P from it) has completed; the MMA issues each P·V as soon as its P is complete.
template <int D, bool COMPACT>
__global__ void __launch_bounds__(tc_threads(COMPACT), COMPACT ? 2 : 1)
    attn_tc_kernel(const __grid_constant__ AttnTcParams tp, __nv_bfloat16* out) {
  constexpr int WPQ = tc_wpq(COMPACT);
  constexpr int kThreads = tc_threads(COMPACT);
  constexpr int kSoftThreads = 128 * WPQ;
  constexpr int kSoftWarps = 4 * WPQ;
  constexpr int HALVES = D / 64;                 // 64-element (128-byte) column blocks of a row
  const int QROWS = COMPACT && p_rows_of(tp) <= 64 ? 64 : kRows;
  const int QH = QROWS * 128;                    // one column block of Q
  constexpr int KH = kKT * 128;                  // one column block of a K or V tile (8 KB)
  constexpr int STAGE = 2 * HALVES * KH;         // K + V of one tile
  constexpr int REC = D + 4;                     // merge record: O, m, l, 2 pad words
  constexpr int SC = kKT / WPQ;                  // S columns per softmax thread (32 or 16)
  constexpr int OC = D / WPQ;                    // O columns per softmax thread
  constexpr int NSB = tc_nsb(COMPACT);           // S/P buffers
  constexpr int kTmemCols = tc_tmem_cols(COMPACT);
  constexpr int kOCol = NSB * kKT;               // O's first TMEM column
  const AttnParams& p = tp.a;
  const int NST = COMPACT ? 2 : tp.stages;

  extern __shared__ uint8_t dsm_raw[];
  __shared__ uint64_t q_full, fin_bar, recv_bar;
  __shared__ uint64_t pv_done[4];   // pv_done[u % NSB]: the P·V of tile u has completed
  __shared__ uint64_t kv_full[kMaxAttnTcStages], kv_empty[kMaxAttnTcStages];
  __shared__ uint64_t s_full[4], p_full[4];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int s_abort;
  __shared__ float red[2][WPQ][kRows];   // [tile parity][column part][row]: partial row maxima, then sums

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = base;
  uint8_t* ring = qs + HALVES * QH;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nr = p.g * p.B;
  int* status = p.status;
  const int kps = attn_kps(p);   // the host's, or the call's device-side plan (global merge)
  int s, h, b;
  if (p.kps_dev) {
    // Device-side plan: the grid is flat, KV head fastest, then the batch's
    // (request, split) items in order, so that the CTAs with keys come first and
    // the ones past the batch's items (launched last) exit at once. Every warp
    // finds its item's request by a scan of the requests' split counts.
    h = blockIdx.x % p.n_kv;
    const int item = blockIdx.x / p.n_kv;
    if (item >= __ldg(p.kps_dev + 1)) return;   // past the batch's items
    b = -1;
    s = 0;
    for (int r0 = 0, before = 0; r0 < p.bs; r0 += 32) {
      const int r = r0 + lane;
      int n = 0;
      if (r < p.bs) {
        int Pr = p.ctx_len[r];
        Pr = Pr < 0 ? 0 : (Pr > p.max_ctx ? p.max_ctx : Pr);
        n = min(p.n_splits, (Pr + p.B - attn_key_base(attn_ctx_lo(Pr, p.window)) + kps - 1) / kps);
      }
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int excl = incl - n;
      const unsigned hit = __ballot_sync(0xffffffffu, r < p.bs && item >= before + excl && item < before + incl);
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (hit) {
        const int src = __ffs((int)hit) - 1;
        b = r0 + src;
        s = item - before - __shfl_sync(0xffffffffu, excl, src);
        break;
      }
      before += total;
    }
    if (b < 0) return;   // past the batch's items
  } else {
    s = blockIdx.x;
    h = blockIdx.y;
    b = blockIdx.z;
  }

  int P = p.ctx_len[b];
  if (P < 0 || P > p.max_ctx) {
    if (threadIdx.x == 0) flag_error(status, ST_BAD_CTX);
    P = P < 0 ? 0 : p.max_ctx;
  }
  // this split's keys: [k0, k1) of the sequence (P context keys, then B block keys),
  // counted from the 64-aligned start of a sliding window (else from 0); context
  // keys below ctx_lo are masked
  const int S = p.n_splits;
  const int T_all = P + p.B;
  const int ctx_lo = attn_ctx_lo(P, p.window);
  const int k0 = min(T_all, attn_key_base(ctx_lo) + s * kps);
  const int k1 = s == S - 1 ? T_all : min(T_all, k0 + kps);
  const int cx1 = min(k1, P);                               // context part [k0, cx1)
  const int n_ctx = cx1 > k0 ? (cx1 - k0 + kKT - 1) / kKT : 0;
  const int bk0 = max(k0, P) - P, bk1 = k1 - P;             // block rows [bk0, bk1)
  const int n_blk = bk1 > bk0 ? (bk1 - bk0 + kKT - 1) / kKT : 0;
  const int n_tiles = n_ctx + n_blk;
  auto tile_valid = [&](int t) {
    return t < n_ctx ? min(kKT, cx1 - (k0 + t * kKT)) : min(kKT, bk1 - (bk0 + (t - n_ctx) * kKT));
  };
  // first valid key column of a tile (non-zero only for the tile holding ctx_lo)
  auto tile_lo = [&](int t) { return t < n_ctx ? max(0, ctx_lo - (k0 + t * kKT)) : 0; };

  const bool gmerge = p.global_merge != 0;
  if (gmerge && n_tiles == 0) return;   // nothing of this request here: the merge kernel skips the split
  const bool cluster = S > 1 && !gmerge;
  const int per = (nr + S - 1) / S;     // merged rows owned by each split (cluster merge)
  const int own_lo = min(nr, s * per), own_hi = min(nr, own_lo + per);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < NSB; ++i) mbar_init(&pv_done[i], 1);
    mbar_init(&fin_bar, 1);
    mbar_init(&recv_bar, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftWarps);   // one arrival per softmax warp
    }
    s_abort = 0;
    fence_mbar_init();
    if (cluster) mbar_arrive_expect_tx(&recv_bar, (uint32_t)(S * (own_hi - own_lo) * REC * 4));
  }
  // The producer (thread 0, which initialised the barriers) issues the first
  // context tiles now, before the block barrier. Context tiles were written by
  // earlier kernels of the stream, all complete by now (every kernel waits for
  // its predecessor before letting its successor start), so they do not wait on
  // the previous kernel either.
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
      const int crow = (page * p.n_kv + h) * p.page_size + kt % p.page_size;
#pragma unroll
      for (int hh = 0; hh < HALVES; ++hh) {
        tma_load_2d(kd + hh * KH, &tp.kcmap, &kv_full[st], hh * 64, crow, pol);
        tma_load_2d(vd + hh * KH, &tp.vcmap, &kv_full[st], hh * 64, crow, pol);
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
  if (threadIdx.x == 0) {
    prefetch_tmap(&tp.kcmap);
    prefetch_tmap(&tp.vcmap);
    prefetch_tmap(&tp.qmap);
    for (int t = 0; t < pre; ++t)
      if (t < n_ctx) issue(t, t);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (QROWS == kRows) {
    // rows nr..127 of Q are padding: zero them (the MMA reads 128 rows)
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

  // softmax threads: warp w owns TMEM lanes 32*(w % 4) .. +31 (one query row per
  // lane) and part (w - 2) / 4 of the key columns; their results stay in
  // registers across the block barrier below
  const int quad = warp & 3;
  const int part = (warp - 2) >> 2;
  const int row = quad * 32 + lane;
  const bool quad_live = quad * 32 < QROWS;       // 64-row Q: lanes 64..127 hold nothing
  const bool active = warp >= 2 && quad_live && row < nr;
  float o[OC];
  float m_used = -INFINITY, l = 0.f;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
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
      auto pv = [&](int u) {   // the caller has seen p_full for tile u
        tc_fence_after();
        const uint32_t vd = smem_addr(ring + (size_t)(u % NST) * STAGE + HALVES * KH);
        // P of tile u sits in its S buffer's first 32 columns (fp16 pairs)
        const uint32_t pa = tmem + (uint32_t)((u % NSB) * kKT);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)   // 16 keys per MMA: +8 columns of P, +2 KB (16 rows) of V
          mma_f16_ts(tmem + kOCol, pa + (uint32_t)(8 * kk), desc_mnmajor_sw128(vd + kk * 2048, KH), id_o,
                     (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&pv_done[u % NSB]);
        mma_commit(&kv_empty[u % NST]);
      };
      bool ok = mbar_wait(&q_full, 0, status);
      // Issue order: the P·V of the oldest softmaxed tile as soon as its P is
      // complete (it frees the tile's ring slot and, once done, its S/P buffer),
      // otherwise the next tile's S once its K/V have landed and the P·V that read
      // its S/P buffer last is complete. Every probe is non-blocking (test_wait:
      // a suspending try_wait on one barrier would hold up work the other allows);
      // the time without progress is bounded.
      int ns = 0, npv = 0;
      uint64_t idle_since = globaltimer_ns();
      while (ok && npv < n_tiles) {
        if (s_abort) {
          ok = false;
          break;
        }
        if (npv < ns && mbar_test_wait(&p_full[npv % NSB], (npv / NSB) & 1)) {
          pv(npv++);
          idle_since = globaltimer_ns();
          continue;
        }
        // the S buffer of tile ns held the P of tile ns - NSB: its P·V must be complete
        if (ns < n_tiles && mbar_test_wait(&kv_full[ns % NST], (ns / NST) & 1) &&
            (ns < NSB || mbar_test_wait(&pv_done[ns % NSB], ((ns - NSB) / NSB) & 1))) {
          tc_fence_after();
          const uint32_t kd = smem_addr(ring + (size_t)(ns % NST) * STAGE);
          const uint32_t qa = smem_addr(qs);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {   // K = d in steps of 16: +32 B inside a 128-byte block
            const int hh = kk >> 2, sub = kk & 3;
            mma_bf16(tmem + (uint32_t)((ns % NSB) * kKT), desc_kmajor_sw128(qa + hh * QH) + (uint64_t)(2 * sub),
                     desc_kmajor_sw128(kd + hh * KH) + (uint64_t)(2 * sub), id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[ns % NSB]);
          ++ns;
          idle_since = globaltimer_ns();
          continue;
        }
        if (globaltimer_ns() - idle_since > kWaitLimitNs) {
          flag_error(status, ST_TIMEOUT);
          ok = false;
        }
      }
      if (!ok) s_abort = 1;
      // every MMA issued has completed before TMEM can be freed
      mma_commit(&fin_bar);
      mbar_wait(&fin_bar, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int tid = threadIdx.x - 64;                            // 0 .. kSoftThreads-1
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = p.scale * 1.4426950408889634f;
    const int c0 = part * SC;                                    // this thread's first key column
    bool ok = true;
    // Every named barrier below is reached by all softmax threads: a failed
    // (timed-out) wait is voted on at the next barrier, and the loop is left by
    // all of them at once.
    for (int t = 0; t < n_tiles; ++t) {
      if (ok) ok = !s_abort && mbar_wait(&s_full[t % NSB], (t / NSB) & 1, status);
      const bool wok = __all_sync(0xffffffffu, ok);
      const int valid = tile_valid(t);
      const int vlo = tile_lo(t);
      float sv[SC];   // raw scores; the max is taken before scaling (sl2 > 0)
      float mx = -INFINITY;
      if (wok && quad_live) {
        tc_fence_after();
        uint32_t sr[SC];
        tmem_ld_cols<SC>(lane_addr + (uint32_t)((t % NSB) * kKT + c0), sr);
        tmem_wait_ld();
        if (valid >= c0 + SC && vlo <= c0) {
#pragma unroll
          for (int c = 0; c < SC; ++c) sv[c] = __uint_as_float(sr[c]);
        } else {
#pragma unroll
          for (int c = 0; c < SC; ++c)
            sv[c] = c0 + c < valid && c0 + c >= vlo ? __uint_as_float(sr[c]) : -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          m8[i] = sv[i];
#pragma unroll
          for (int j = i + 8; j < SC; j += 8) m8[i] = fmaxf(m8[i], sv[j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) m8[i] = fmaxf(m8[i], m8[i + 4]);
        mx = fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])) * sl2;
      }
      // the row's tile max over all its column parts; the same barrier votes on
      // failure, and orders every thread's S reads before any P write into the buffer
      red[t & 1][part][row] = mx;
      if (named_bar_or(1, kSoftThreads, !wok)) {
        ok = false;
        s_abort = 1;
        break;
      }
#pragma unroll
      for (int q2 = 0; q2 < WPQ; ++q2) mx = fmaxf(mx, red[t & 1][q2][row]);
      float alpha = 1.f;
      bool resc = false;
      if (m_used == -INFINITY) {
        m_used = mx;   // first keys of this row: nothing accumulated yet
      } else if (mx > m_used + kLazyLog2) {
        alpha = ex2(m_used - mx);
        m_used = mx;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc && quad_live)) {
        // O holds tiles < t: wait for the P·V of tile t-1, then rescale this thread's O columns
        if (ok) ok = mbar_wait(&pv_done[(t - 1) % NSB], ((t - 1) / NSB) & 1, status);
        if (__all_sync(0xffffffffu, ok)) {
          tc_fence_after();
          constexpr int CH = OC < 32 ? OC : 32;   // in pieces, to keep registers for the scores
#pragma unroll 1
          for (int cc = 0; cc < OC; cc += CH) {
            uint32_t r[CH];
            tmem_ld_cols<CH>(lane_addr + (uint32_t)(kOCol + part * OC + cc), r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < CH; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st_cols<CH>(lane_addr + (uint32_t)(kOCol + part * OC + cc), r);
          }
          tmem_wait_st();
        }
        l *= alpha;
      }
      if (quad_live) {
        // P (fp16, <= 2^8) as fp16 pairs into the first 32 columns of this tile's S
        // buffer: this thread's keys c0 .. c0+SC-1 are columns c0/2 .. c0/2+SC/2-1.
        // A row with no key yet has m_used = -inf and only masked scores (-inf):
        // subtracting 0 instead keeps 2^(-inf) = 0.
        const float mneg = m_used == -INFINITY ? 0.f : -m_used;
        uint32_t pk[SC / 2];
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < SC; c += 2) {
          const float e0 = ex2(fmaf(sv[c], sl2, mneg)), e1 = ex2(fmaf(sv[c + 1], sl2, mneg));
          ps[(c >> 1) & 3] += e0 + e1;
          pk[c >> 1] = pack_f16x2(e0, e1);
        }
        tmem_st_cols<SC / 2>(lane_addr + (uint32_t)((t % NSB) * kKT + c0 / 2), pk);
        tmem_wait_st();
        l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      }
      // a partial tile: V rows outside the valid keys may hold anything (even NaN,
      // which a zero probability would not cancel); zero them
      if (valid < kKT || vlo > 0) {
        uint8_t* vd = ring + (size_t)(t % NST) * STAGE + HALVES * KH;
        const int n_hi = (kKT - valid) * 8, n = n_hi + vlo * 8;   // 16-byte chunks per column block
        for (int e = tid; e < n * HALVES; e += kSoftThreads) {
          const int hh = e / n, c = e % n;
          const int off = c < n_hi ? valid * 128 + c * 16 : (c - n_hi) * 16;
          *reinterpret_cast<uint4*>(vd + hh * KH + off) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();   // the zeroed V rows, for the MMA
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t % NSB]);
    }
    // final O columns of this thread; the row's sum over all its column parts
    bool have = ok && n_tiles > 0;
    if (have) have = mbar_wait(&pv_done[(n_tiles - 1) % NSB], ((n_tiles - 1) / NSB) & 1, status);
    if (__all_sync(0xffffffffu, have)) {
      if (quad_live) {
        tc_fence_after();
        uint32_t r[OC];
        tmem_ld_cols<OC>(lane_addr + (uint32_t)(kOCol + part * OC), r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < OC; ++i) o[i] = __uint_as_float(r[i]);
      }
    } else {
      if (n_tiles > 0) s_abort = 1;
#pragma unroll
      for (int c = 0; c < OC; ++c) o[c] = 0.f;
      m_used = -INFINITY;
      l = 0.f;
    }
    // (the slot parity the last tile's max exchange did not use)
    red[n_tiles & 1][part][row] = l;
    named_bar_sync(1, kSoftThreads);
    l = 0.f;
#pragma unroll
    for (int q2 = 0; q2 < WPQ; ++q2) l += red[n_tiles & 1][q2][row];
  }
  tc_fence_before();
  __syncthreads();   // ring, Q and TMEM are dead for every role
  if (cluster) cluster_arrive_release();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (active) {
    const int i_blk = row / p.g, j_head = row % p.g;   // TMA wrote Q rows in (block row, head) order
    if (gmerge) {
      const size_t pr = ((size_t)(b * p.n_kv + h) * S + s) * nr + (size_t)j_head * p.B + i_blk;
      float* po = p.part_o + pr * D + part * OC;
#pragma unroll
      for (int c = 0; c < OC; c += 4) *reinterpret_cast<float4*>(po + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      if (part == 0) {
        p.part_m[pr] = m_used;
        p.part_l[pr] = l;
      }
    } else if (!cluster) {
      const float inv = 1.f / l;
      __nv_bfloat16* dst =
          out + (size_t)(b * p.B + i_blk) * (p.n_q * D) + (size_t)(h * p.g + j_head) * D + part * OC;
#pragma unroll
      for (int c = 0; c < OC; c += 8) {
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
    } else {
      float* rec = reinterpret_cast<float*>(base) + (size_t)row * REC;
#pragma unroll
      for (int c = 0; c < OC; c += 4)
        *reinterpret_cast<float4*>(rec + part * OC + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      if (part == 0) {
        rec[D] = m_used;
        rec[D + 1] = l;
      }
    }
  }
  if (!cluster) return;

  // ---- cluster merge: each owner gets every split's records of its rows
  float* stg = reinterpret_cast<float*>(base);
  float* rcv = stg + (size_t)nr * REC;
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
    const float w = (lane < S && ms != -INFINITY) ? ex2(ms - M) : 0.f;
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

size_t attn_tc_smem_bytes(int d, bool compact, int stages, int splits, bool gmerge, int nr) {
  const int halves = d / 64;
  const int qrows = compact && nr <= 64 ? 64 : kRows;
  const int nst = compact ? 2 : stages;
  const size_t loads = (size_t)halves * qrows * 128 + (size_t)nst * 2 * halves * kKT * 128;
  const size_t rec = (size_t)(d + 4) * 4;
  const size_t per = (size_t)(nr + splits - 1) / splits;
  const size_t merge = splits > 1 && !gmerge ? ((size_t)nr + (size_t)splits * per) * rec : 0;
  return (loads > merge ? loads : merge) + 1024;
}

static const void* attn_tc_fn(int d, bool compact) {
  if (d == 128) return compact ? (const void*)attn_tc_kernel<128, true> : (const void*)attn_tc_kernel<128, false>;
  return compact ? (const void*)attn_tc_kernel<64, true> : (const void*)attn_tc_kernel<64, false>;
}

// Raise the kernel's dynamic shared-memory limit (once per size) and allow 16-CTA clusters.
static cudaError_t attn_tc_prepare(int d, bool compact, size_t smem) {
  static size_t set[4] = {0, 0, 0, 0};
  const int k = (d == 128 ? 2 : 0) + (compact ? 1 : 0);
  if (smem <= set[k]) return cudaSuccess;
  const void* fn = attn_tc_fn(d, compact);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  // all of the unified L1 / shared memory as shared memory, so that two compact CTAs fit
  e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  set[k] = smem;
  return cudaSuccess;
}

cudaError_t launch_attn_tc(const AttnTcParams& tp, void* out, cudaStream_t st, bool pdl) {
  const AttnParams& p = tp.a;
  if (p.n_splits < 1 || (!p.global_merge && p.n_splits > kMaxAttnCluster) || p.kps % kKT || p.page_size % kKT)
    return cudaErrorInvalidValue;
  if (tp.stages < 2 || tp.stages > kMaxAttnTcStages || p.g * p.B > kRows || (p.d != 64 && p.d != 128))
    return cudaErrorInvalidValue;
  const bool compact = tp.compact != 0;
  const bool gmerge = p.global_merge != 0;
  const size_t smem = attn_tc_smem_bytes(p.d, compact, tp.stages, p.n_splits, gmerge, p.g * p.B);
  cudaError_t e = attn_tc_prepare(p.d, compact, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  // device-side plan: one flat grid over (request, split) items x KV heads
  cfg.gridDim = p.kps_dev ? dim3((unsigned)(p.n_splits * p.n_kv * p.bs), 1, 1) : dim3(p.n_splits, p.n_kv, p.bs);
  cfg.blockDim = dim3(tc_threads(compact));
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
  return cudaLaunchKernelExC(&cfg, attn_tc_fn(p.d, compact), args);
}

// Clusters of n CTAs (n = 1: single CTAs) of this kernel's shape that can be resident at once (0: none fit).
int attn_tc_max_clusters(int d, bool compact, int stages, int n, bool gmerge, int nr) {
  const size_t smem = attn_tc_smem_bytes(d, compact, stages, n, gmerge, nr);
  if (attn_tc_prepare(d, compact, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n, 1, 1);
  cfg.blockDim = dim3(tc_threads(compact));
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)n;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int num = 0;
  if (cudaOccupancyMaxActiveClusters(&num, attn_tc_fn(d, compact), &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return num;
}

}  // namespace dfl
