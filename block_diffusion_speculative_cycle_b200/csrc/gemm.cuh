// Skinny "weight-streaming" GEMM of the draft cycle: D = X · Wᵀ where W is a
// stack of weight segments ([rows, K] each, bf16/fp32, K contiguous) and X the
// activation rows ([M, K]). The output tile is 128 weight rows x up to 256
// activation rows; its epilogue is fused (see EpiKind).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "philox.cuh"

namespace dfl {

constexpr int kMaxSeg = 16;      // weight segments per launch
constexpr int kTileN = 128;      // weight rows per output tile
constexpr int kChunkRows = 32;   // activation rows per epilogue chunk
constexpr int kChunkLd = 129;    // padded row stride of the epilogue staging tile (floats)

enum EpiKind : int {
  EPI_STORE = 0,      // out[s][m, n] = acc                              (fusion projection c)
  EPI_QKV = 1,        // q / k / v of the block rows, RoPE on flagged segments
  EPI_KV_INJECT = 2,  // injected K (RoPE) / V scattered into each layer's cache pages
  EPI_RESID = 3,      // x[m, n] += acc                                  (Wo, Wdown)
  EPI_SWIGLU = 4,     // act[m, f] = silu(gate) * up (paired gate/up tiles)
  EPI_ARGMAX = 5,     // per activation row, max over the tile's vocab rows -> keys[m]
  EPI_SAMPLE = 6,     // Gumbel-max draw per row (keys[m]) + the row's logits stored
};

struct EpiParams {
  int kind;
  int n_seg;
  int seg_tile_begin[kMaxSeg + 1];   // first output tile of each segment; [n_seg] = total tiles
  void* out[kMaxSeg];                // per-segment destination (buffer or cache page pool)
  int ld_out[kMaxSeg];               // leading dimension (elements) of out[s] for STORE/QKV/SWIGLU
  unsigned int rope_mask;            // bit s: rotate segment s
  int head_dim;
  const double* inv_freq;            // [head_dim/2] theta^(-2i/d), double
  const float2* rope_cs;             // [rows][head_dim/2] (cos, sin) of each activation row's position
  RopeFill fill;                     // side job of this launch: fill the next launch's RoPE table
  int rows_per_req;                  // activation row m belongs to request m / rows_per_req
  const int* pos_base;               // [bs] absolute position of each request's first row
  const int* row_count;              // [bs] valid rows per request (nullptr: all)
  const int* page_table;             // [bs, max_pages]
  int max_pages, num_pages, page_size, n_kv;
  int cache_type;                    // element type of the KV cache pools (OUT_F32 / OUT_BF16 / OUT_F16)
  float* x;                          // residual stream [M, ldx] fp32
  int ldx;
  // Deferred RMSNorm of this GEMM's input rows (the input is x ⊙ gain, not yet
  // normalised): acc *= rsqrt(sum_p norm_part[p * ld_part + row] / H + eps),
  // the partial sums of squares summed in p order. Null: input already normalised.
  const float* norm_part;
  int n_part, ld_part;
  float norm_inv_h, norm_eps;
  // Residual epilogue extras: the next norm's operand xg = x_new ⊙ gamma_next
  // (model dtype, [M, ldx]) and this tile's partial sums of squares of x_new,
  // sumsq[tile * ld_part + row]. Null: not produced.
  const float* gamma_next;
  void* xg;
  float* sumsq;
  unsigned long long* keys;          // [M] packed argmax keys
  // EPI_SAMPLE: row m = request m / rows_per_req, block position i = m % rows_per_req;
  // rows with i >= 1 draw argmax_v (logit / T + Gumbel noise) into keys[m] and store
  // their logits (fp32) at logits_out[(req * (rows_per_req - 1) + i - 1) * ld_logits + v].
  float inv_temp;
  uint32_t seed_lo, seed_hi;
  float* logits_out;
  int ld_logits;
  int* status;
  int out_type;                      // OUT_F32 / OUT_BF16 / OUT_F16 / OUT_BF16X2 (see store_out)
  size_t out_plane;                  // OUT_BF16X2: elements from the hi plane to the lo plane
};

__device__ __forceinline__ int seg_of_tile(const EpiParams& e, int tile) {
  int s = 0;
  while (s + 1 < e.n_seg && e.seg_tile_begin[s + 1] <= tile) ++s;
  return s;
}

// Output element types. OUT_BF16X2 stores v as a pair of bf16 planes: hi = bf16(v)
// at idx and lo = bf16(v - hi) at idx + plane, so that a GEMM reading both planes
// as operands sees v to about 16 significant bits.
enum OutType : int { OUT_F32 = 0, OUT_BF16 = 1, OUT_F16 = 2, OUT_BF16X2 = 3 };

__device__ __forceinline__ void store_out(void* base, size_t idx, float v, int type, size_t plane = 0) {
  switch (type) {
    case OUT_BF16:
      reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
      break;
    case OUT_F16:
      reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
      break;
    case OUT_BF16X2: {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      reinterpret_cast<__nv_bfloat16*>(base)[idx] = hi;
      reinterpret_cast<__nv_bfloat16*>(base)[idx + plane] = __float2bfloat16_rn(v - __bfloat162float(hi));
      break;
    }
    default:
      reinterpret_cast<float*>(base)[idx] = v;
  }
}

// Scratch of the epilogue (shared memory, per CTA): row scales, then an 8 x 32-float
// reduction area (4 x 32 floats, or 4 x 32 64-bit argmax keys).
constexpr int kEpiScratch = kChunkRows + 8 * kChunkRows;

// Row scales of the deferred RMSNorm for rows row0 .. row0+nrows-1 into
// scale[0..nrows): warp w takes rows w, w+4, ...; lane i sums partials i,
// i+32, ... and a butterfly reduction (fixed order, so the result is the same
// on every run) totals the row. Eight rows' loads are issued before any sum.
// Called by the 128 epilogue threads; the caller synchronises them before the
// epilogue reads the scales.
__device__ __forceinline__ void epilogue_row_scales(const EpiParams& e, int row0, int nrows, float* scale, int t) {
  if (!e.norm_part) return;
  const int w = t >> 5, lane = t & 31;
  for (int base = 0; base < nrows; base += 32) {
    float v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = base + w + 4 * r;
      float s = 0.f;
      if (j < nrows)
        for (int i = lane; i < e.n_part; i += 32) s += __ldcg(e.norm_part + (size_t)i * e.ld_part + row0 + j);
      v[r] = s;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = base + w + 4 * r;
      const float ss = warp_sum(v[r]);
      if (j < nrows && lane == 0) scale[j] = rsqrtf(ss * e.norm_inv_h + e.norm_eps);
    }
  }
}

// Apply the epilogue of kind KIND to one staged chunk: acc[j * kChunkLd + t]
// holds the accumulator of activation row row0 + j (j < nrows) and tile row t
// (0..127), scaled by rs[j] when the input rows carry a deferred norm (rs is
// ignored otherwise); the residual epilogue overwrites it. red is a
// [8][kChunkRows]-float scratch area (8-byte aligned). Called by 128 threads with
// t = their tile row; the residual, argmax and (wide) injection epilogues
// synchronise the 128 threads (named barrier 2).
// Each of the four epilogue warps runs alone on its scheduler. A chunk of a few
// rows (the rows one split owns in a split-K cluster) takes a small rolled loop:
// the code is fetched cold once per CTA and its size sets the time. Wider chunks
// take kEpiU rows at a time with their loads and long-latency arithmetic issued
// before any result is used, so no row waits out a full memory or math latency
// on its own.
constexpr int kEpiNarrow = 8;
constexpr int kEpiU = 8;

template <int KIND>
__device__ inline void epilogue_chunk_k(const EpiParams& e, int tile, int row0, int nrows, float* acc, int t,
                                        const float* rs, float* red) {
  if (!e.norm_part) rs = nullptr;
  // The launch parameters live in constant memory and are reached through a
  // reference: copy what the row loops use into registers once, so no global
  // store inside a loop can force them to be read again.
  const int out_type = e.out_type;
  const size_t out_plane = e.out_plane;
  const int rpr = e.rows_per_req;
  const int* const pos_base = e.pos_base;
  auto A = [&](int j, int c) -> float {
    const float v = acc[j * kChunkLd + c];
    return rs ? v * rs[j] : v;
  };
  if constexpr (KIND == EPI_STORE || KIND == EPI_QKV) {
    const int s = seg_of_tile(e, tile);
    const int n = (tile - e.seg_tile_begin[s]) * kTileN + t;
    const bool rope = KIND == EPI_QKV && ((e.rope_mask >> s) & 1u);
    const int d = e.head_dim, half = d >> 1;
    const int jd = n % d;
    const int tp = jd < half ? t + half : t - half;
    // (cos, sin) of row m at this thread's frequency: the call's RoPE table
    const float2* const cs_col = e.rope_cs + jd % half;
    void* const out = e.out[s];
    const size_t ld = (size_t)e.ld_out[s];
    if (nrows <= kEpiNarrow) {
#pragma unroll 1
      for (int j = 0; j < nrows; ++j) {
        const int m = row0 + j;
        float v = A(j, t);
        if (rope) {
          const float2 r = __ldg(cs_col + (size_t)m * half);
          const float w = A(j, tp);
          v = jd < half ? v * r.x - w * r.y : v * r.x + w * r.y;
        }
        store_out(out, (size_t)m * ld + n, v, out_type, out_plane);
      }
      return;
    }
#pragma unroll 1
    for (int j0 = 0; j0 < nrows; j0 += kEpiU) {
      float2 r[kEpiU];
      if (rope) {
#pragma unroll
        for (int u = 0; u < kEpiU; ++u) r[u] = __ldg(cs_col + (size_t)(row0 + min(j0 + u, nrows - 1)) * half);
      }
#pragma unroll
      for (int u = 0; u < kEpiU; ++u) {
        const int j = j0 + u;
        if (j < nrows) {
          float v = A(j, t);
          if (rope) {
            const float w = A(j, tp);
            v = jd < half ? v * r[u].x - w * r[u].y : v * r[u].x + w * r[u].y;
          }
          store_out(out, (size_t)(row0 + j) * ld + n, v, out_type, out_plane);
        }
      }
    }
  } else if constexpr (KIND == EPI_KV_INJECT) {
    const int s = seg_of_tile(e, tile);
    const int n = (tile - e.seg_tile_begin[s]) * kTileN + t;
    const bool rope = (e.rope_mask >> s) & 1u;
    const int d = e.head_dim, half = d >> 1;
    const int jd = n % d, head = n / d;
    const int tp = jd < half ? t + half : t - half;
    const float2* const cs_col = e.rope_cs + jd % half;   // the call's RoPE table, this frequency
    void* const out = e.out[s];
    const int cache_type = e.cache_type;
    const int* const row_count = e.row_count;
    const int* const page_table = e.page_table;
    const int max_pages = e.max_pages, num_pages = e.num_pages, page_size = e.page_size, n_kv = e.n_kv;
    int* const status = e.status;
    // destination of row j (-1: not stored; a bad position or page is flagged by
    // the thread that has `flag`)
    auto dest = [&](int j, int* pos_out, bool flag) -> long long {
      const int m = row0 + j;
      const int req = m / rpr, i = m % rpr;
      if (j >= nrows || (row_count && i >= __ldg(row_count + req))) return -1;
      const int ps = __ldg(pos_base + req) + i;
      const int slot = ps / page_size;
      if (ps < 0 || slot >= max_pages) {
        if (flag) flag_error(status, ST_BAD_PAGE);
        return -1;
      }
      const int page = __ldg(page_table + (size_t)req * max_pages + slot);
      if (page < 0 || page >= num_pages) {
        if (flag) flag_error(status, ST_BAD_PAGE);
        return -1;
      }
      *pos_out = ps;
      return (long long)((((size_t)page * n_kv + head) * page_size + (ps % page_size)) * d + jd);
    };
    if (nrows <= kEpiNarrow) {
#pragma unroll 1
      for (int j = 0; j < nrows; ++j) {
        int ps = 0;
        const long long dst = dest(j, &ps, t == 0);
        if (dst < 0) continue;
        float v = A(j, t);
        if (rope) {
          const float2 r = __ldg(cs_col + (size_t)(row0 + j) * half);
          const float w = A(j, tp);
          v = jd < half ? v * r.x - w * r.y : v * r.x + w * r.y;
        }
        store_out(out, (size_t)dst, v, cache_type);
      }
      return;
    }
    // Wider chunks: thread t < nrows finds row t's cache slot once for all 128
    // columns (the head's offset added per thread), through shared memory
    long long* slot_of = reinterpret_cast<long long*>(red);   // [kChunkRows]; -1: not stored
    if (t < nrows) {
      int ps = 0;
      const long long d0 = dest(t, &ps, true);   // this thread's column: head, jd
      slot_of[t] = d0 < 0 ? -1 : d0 - ((long long)head * page_size * d + jd);
    }
    asm volatile("bar.sync 2, 128;" ::: "memory");
    const long long col = (long long)head * page_size * d + jd;
#pragma unroll 1
    for (int j0 = 0; j0 < nrows; j0 += kEpiU) {
      // destination of each row (-1: not stored), then the rotation
      long long dst[kEpiU];
#pragma unroll
      for (int u = 0; u < kEpiU; ++u) {
        const long long sl = j0 + u < nrows ? slot_of[j0 + u] : -1;
        dst[u] = sl < 0 ? -1 : sl + col;
      }
      float2 r[kEpiU];
      if (rope) {
#pragma unroll
        for (int u = 0; u < kEpiU; ++u) r[u] = __ldg(cs_col + (size_t)(row0 + min(j0 + u, nrows - 1)) * half);
      }
#pragma unroll
      for (int u = 0; u < kEpiU; ++u) {
        if (dst[u] < 0) continue;
        const int j = j0 + u;
        float v = A(j, t);
        if (rope) {
          const float w = A(j, tp);
          v = jd < half ? v * r[u].x - w * r[u].y : v * r[u].x + w * r[u].y;
        }
        store_out(out, (size_t)dst[u], v, cache_type);
      }
    }
  } else if constexpr (KIND == EPI_RESID) {
    const int n = tile * kTileN + t;
    const int w = t >> 5, lane = t & 31;
    float* const x = e.x;
    const size_t ldx = (size_t)e.ldx;
    void* const xg = e.xg;
    float* const sumsq = e.sumsq;
    const float gn = xg ? __ldg(e.gamma_next + n) : 0.f;
    if (nrows <= kEpiNarrow) {
#pragma unroll 1
      for (int j = 0; j < nrows; ++j) {
        float* xp = x + (size_t)(row0 + j) * ldx + n;
        const float xv = *xp + A(j, t);
        *xp = xv;
        if (xg) store_out(xg, (size_t)(row0 + j) * ldx + n, xv * gn, out_type, out_plane);
        if (sumsq) {
          const float ss = warp_sum(xv * xv);
          if (lane == 0) red[w * kChunkRows + j] = ss;
        }
      }
    } else {
      // every row's residual first (independent loads), then add and store; the
      // squares go back into this thread's own staging slots for the row sums
      float xo[kChunkRows];
#pragma unroll
      for (int j = 0; j < kChunkRows; ++j) xo[j] = j < nrows ? x[(size_t)(row0 + j) * ldx + n] : 0.f;
#pragma unroll
      for (int j = 0; j < kChunkRows; ++j) {
        if (j < nrows) {
          const float xv = xo[j] + A(j, t);
          x[(size_t)(row0 + j) * ldx + n] = xv;
          if (xg) store_out(xg, (size_t)(row0 + j) * ldx + n, xv * gn, out_type, out_plane);
          acc[j * kChunkLd + t] = xv * xv;
        }
      }
      if (sumsq) {
        // warp w sums columns 32w .. 32w+31 of row `lane` in column order
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (lane < nrows) {
          const float* r = acc + lane * kChunkLd + 32 * w;
          float ss = 0.f;
#pragma unroll 8
          for (int c = 0; c < 32; ++c) ss += r[c];
          red[w * kChunkRows + lane] = ss;
        }
      }
    }
    if (sumsq) {
      // this tile's 128 columns of each row: the 4 warp sums in warp order
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (t < nrows)
        sumsq[(size_t)tile * e.ld_part + row0 + t] =
            red[t] + red[kChunkRows + t] + red[2 * kChunkRows + t] + red[3 * kChunkRows + t];
    }
  } else if constexpr (KIND == EPI_SWIGLU) {
    // column c of the 64 gate / up pairs; the two thread halves take alternate rows
    const int c = t & (kTileN / 2 - 1);
    const int f = tile * (kTileN / 2) + c;
    void* const out = e.out[0];
    const size_t ld = (size_t)e.ld_out[0];
#pragma unroll kEpiU
    for (int j = t >> 6; j < nrows; j += 2) {
      const float g = A(j, c), u = A(j, c + kTileN / 2);
      store_out(out, (size_t)(row0 + j) * ld + f, silu_f(g) * u, out_type, out_plane);
    }
  } else if constexpr (KIND == EPI_SAMPLE) {
    // warp w takes rows w, w+4, ...; lane scans vocab rows vbase + lane + 32k, k < 4,
    // whose uniforms are the four words of one Philox block at counter
    // (tile, lane, i, req): the draft-noise layout of the sampled drafter
    const int w = t >> 5, lane = t & 31;
    const int vbase = tile * kTileN;
#pragma unroll 1
    for (int j = w; j < nrows; j += 4) {
      const int m = row0 + j;
      const int req = m / e.rows_per_req, i = m % e.rows_per_req;
      if (i == 0) continue;   // the anchor row drafts nothing
      const uint4 r = philox4x32_10(make_uint4((uint32_t)tile, (uint32_t)lane, (uint32_t)i, (uint32_t)req), e.seed_lo,
                                    e.seed_hi);
      const uint32_t words[4] = {r.x, r.y, r.z, r.w};
      float* lo = e.logits_out + ((size_t)req * (e.rows_per_req - 1) + i - 1) * e.ld_logits + vbase;
      unsigned long long best = 0ull;
#pragma unroll
      for (int k = 0; k < kTileN / 32; ++k) {
        const int c = lane + 32 * k;
        const float logit = A(j, c);
        lo[c] = logit;
        const float gumbel = -logf(-logf(philox_uniform(words[k])));
        const unsigned long long key = argmax_key(fmaf(logit, e.inv_temp, gumbel), vbase + c);
        best = key > best ? key : best;
      }
      best = warp_max_u64(best);
      if (lane == 0) atomicMax(e.keys + m, best);
    }
  } else if constexpr (KIND == EPI_ARGMAX) {
    // lane = row of the chunk, warp w = vocab rows 32w .. 32w+31 of the tile (no
    // shuffles: each thread scans its 32 scores), then the 4 warps' keys of a row
    // meet in shared memory and one thread per row folds them into keys[m]
    const int w = t >> 5, lane = t & 31;
    const int vbase = tile * kTileN + 32 * w;
    unsigned long long* red64 = reinterpret_cast<unsigned long long*>(red);
    if (lane < nrows) {
      const float* row = acc + lane * kChunkLd + 32 * w;
      const float sc = rs ? rs[lane] : 1.f;
      unsigned long long best = 0ull;
#pragma unroll 8
      for (int c = 0; c < 32; ++c) {
        const float v = rs ? row[c] * sc : row[c];
        const unsigned long long key = argmax_key(v, vbase + c);
        best = key > best ? key : best;
      }
      red64[w * kChunkRows + lane] = best;
    }
    asm volatile("bar.sync 2, 128;" ::: "memory");
    if (t < nrows) {
      unsigned long long best = red64[t];
#pragma unroll
      for (int q = 1; q < 4; ++q) best = red64[q * kChunkRows + t] > best ? red64[q * kChunkRows + t] : best;
      atomicMax(e.keys + row0 + t, best);
    }
  }
}

// Runtime dispatch (CUDA-core GEMM): scratch[0..kChunkRows) holds the row scales,
// the rest the reduction area.
__device__ inline void epilogue_chunk(const EpiParams& e, int tile, int row0, int nrows, float* acc, int t,
                                      float* scratch) {
  const float* rs = scratch;
  float* red = scratch + kChunkRows;
  switch (e.kind) {
    case EPI_STORE: epilogue_chunk_k<EPI_STORE>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_QKV: epilogue_chunk_k<EPI_QKV>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_KV_INJECT: epilogue_chunk_k<EPI_KV_INJECT>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_RESID: epilogue_chunk_k<EPI_RESID>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_SWIGLU: epilogue_chunk_k<EPI_SWIGLU>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_ARGMAX: epilogue_chunk_k<EPI_ARGMAX>(e, tile, row0, nrows, acc, t, rs, red); break;
    case EPI_SAMPLE: epilogue_chunk_k<EPI_SAMPLE>(e, tile, row0, nrows, acc, t, rs, red); break;
    default: break;
  }
}

// ---------------------------------------------------------------- launch descriptions
struct GemmSimtParams {
  const void* w[kMaxSeg];   // weight segment bases
  int paired;               // tile = 64 rows of w[0] + the same 64 rows of w[1]
  const void* x;            // activations [M, ldx]
  int ldx;
  int M, K;
  int w_bf16, x_bf16;
  size_t x_plane;           // bf16 split activations: elements to the lo plane (0: single plane)
  EpiParams epi;
};

struct alignas(64) GemmTcParams {
  CUtensorMap wmap[kMaxSeg];   // weight segment maps: box 64 (K) x 128 rows (64 rows when paired)
  CUtensorMap xmap;            // activation map: box 64 (K) x m_tile rows (both planes when x_split)
  EpiParams epi;
  int paired;
  int M;                       // valid activation rows
  int m_tile;                  // activation rows per CTA (multiple of 16; MMA N = (1 + x_split) * m_tile <= 256)
  int x_split;                 // activations are hi/lo bf16 planes; the lo plane starts x_plane_rows rows on
  int x_plane_rows;
  int m_blocks;
  int tmem_cols;
  int num_kb;                  // K / 64
  int splits;                  // K splits = cluster size (1..8)
  int kb_per_split;
  int n_tiles;
  int stages;
  int use_pdl;
  // Failure-injection hook, 0 in normal use: when set, every epilogue thread,
  // once the accumulator is final, also waits on a barrier nothing ever arrives
  // at, bounded by this many ns, so the bounded-wait give-up path runs (ST_TIMEOUT
  // flagged, epilogue skipped, TMEM freed) with no copy or MMA in flight.
  unsigned int test_stall_ns;
};

cudaError_t launch_gemm_simt(const GemmSimtParams& p, int n_tiles, cudaStream_t st, bool pdl);
cudaError_t launch_gemm_tc(const GemmTcParams& p, cudaStream_t st);
size_t gemm_tc_smem_bytes(int m_tile, int x_split, int stages, int splits);
constexpr int kMaxClusterSplits = 8;

}  // namespace dfl
