// Skinny "weight-streaming" GEMM of the draft cycle: D = X · Wᵀ where W is a
// stack of weight segments ([rows, K] each, bf16/fp32, K contiguous) and X the
// activation rows ([M, K]). The output tile is 128 weight rows x up to 256
// activation rows; its epilogue is fused (see EpiKind).
#pragma once

#include "common.cuh"

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
};

struct EpiParams {
  int kind;
  int n_seg;
  int seg_tile_begin[kMaxSeg + 1];   // first output tile of each segment; [n_seg] = total tiles
  void* out[kMaxSeg];                // per-segment destination (buffer or cache page pool)
  int ld_out[kMaxSeg];               // leading dimension (elements) of out[s] for STORE/QKV/SWIGLU
  unsigned int rope_mask;            // bit s: rotate segment s
  int head_dim;
  double log2_theta;
  int rows_per_req;                  // activation row m belongs to request m / rows_per_req
  const int* pos_base;               // [bs] absolute position of each request's first row
  const int* row_count;              // [bs] valid rows per request (nullptr: all)
  const int* page_table;             // [bs, max_pages]
  int max_pages, num_pages, page_size, n_kv;
  float* x;                          // residual stream [M, ldx] fp32
  int ldx;
  unsigned long long* keys;          // [M] packed argmax keys
  int* status;
  int out_bf16;                      // 1: bf16 outputs, 0: fp32 outputs
};

__device__ __forceinline__ int seg_of_tile(const EpiParams& e, int tile) {
  int s = 0;
  while (s + 1 < e.n_seg && e.seg_tile_begin[s + 1] <= tile) ++s;
  return s;
}

__device__ __forceinline__ void store_out(void* base, size_t idx, float v, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(base)[idx] = v;
}

// Apply the epilogue to one staged chunk: acc[j * kChunkLd + t] holds the
// accumulator of activation row row0 + j (j < nrows) and tile row t (0..127).
// Called by 128 threads with t = their tile row; no barrier inside.
__device__ inline void epilogue_chunk(const EpiParams& e, int tile, int row0, int nrows, const float* acc, int t) {
  switch (e.kind) {
    case EPI_STORE:
    case EPI_QKV: {
      const int s = seg_of_tile(e, tile);
      const int n = (tile - e.seg_tile_begin[s]) * kTileN + t;
      const bool rope = (e.rope_mask >> s) & 1u;
      const int d = e.head_dim, half = d >> 1;
      const int jd = n % d;
      const int tp = jd < half ? t + half : t - half;
      for (int j = 0; j < nrows; ++j) {
        const int m = row0 + j;
        float v = acc[j * kChunkLd + t];
        if (rope) {
          const int req = m / e.rows_per_req, i = m % e.rows_per_req;
          const int pos = e.pos_base[req] + i;
          float c, sn;
          rope_cos_sin(pos, jd % half, d, e.log2_theta, &c, &sn);
          const float w = acc[j * kChunkLd + tp];
          v = jd < half ? v * c - w * sn : v * c + w * sn;
        }
        store_out(e.out[s], (size_t)m * e.ld_out[s] + n, v, e.out_bf16);
      }
      break;
    }
    case EPI_KV_INJECT: {
      const int s = seg_of_tile(e, tile);
      const int n = (tile - e.seg_tile_begin[s]) * kTileN + t;
      const bool rope = (e.rope_mask >> s) & 1u;
      const int d = e.head_dim, half = d >> 1;
      const int jd = n % d, head = n / d;
      const int tp = jd < half ? t + half : t - half;
      for (int j = 0; j < nrows; ++j) {
        const int m = row0 + j;
        const int req = m / e.rows_per_req, i = m % e.rows_per_req;
        if (e.row_count && i >= e.row_count[req]) continue;
        const int pos = e.pos_base[req] + i;
        const int slot = pos / e.page_size;
        if (pos < 0 || slot >= e.max_pages) {
          if (t == 0) flag_error(e.status, ST_BAD_PAGE);
          continue;
        }
        const int page = e.page_table[(size_t)req * e.max_pages + slot];
        if (page < 0 || page >= e.num_pages) {
          if (t == 0) flag_error(e.status, ST_BAD_PAGE);
          continue;
        }
        float v = acc[j * kChunkLd + t];
        if (rope) {
          float c, sn;
          rope_cos_sin(pos, jd % half, d, e.log2_theta, &c, &sn);
          const float w = acc[j * kChunkLd + tp];
          v = jd < half ? v * c - w * sn : v * c + w * sn;
        }
        const size_t dst = (((size_t)page * e.n_kv + head) * e.page_size + (pos % e.page_size)) * d + jd;
        store_out(e.out[s], dst, v, e.out_bf16);
      }
      break;
    }
    case EPI_RESID: {
      const int n = tile * kTileN + t;
      for (int j = 0; j < nrows; ++j) e.x[(size_t)(row0 + j) * e.ldx + n] += acc[j * kChunkLd + t];
      break;
    }
    case EPI_SWIGLU: {
      if (t < kTileN / 2) {
        const int f = tile * (kTileN / 2) + t;
        for (int j = 0; j < nrows; ++j) {
          const float g = acc[j * kChunkLd + t], u = acc[j * kChunkLd + t + kTileN / 2];
          store_out(e.out[0], (size_t)(row0 + j) * e.ld_out[0] + f, silu_f(g) * u, e.out_bf16);
        }
      }
      break;
    }
    case EPI_ARGMAX: {
      if (t < nrows) {
        const int vbase = tile * kTileN;
        unsigned long long best = 0ull;
        for (int c = 0; c < kTileN; ++c) {
          const unsigned long long k = argmax_key(acc[t * kChunkLd + c], vbase + c);
          best = k > best ? k : best;
        }
        atomicMax(e.keys + row0 + t, best);
      }
      break;
    }
    default:
      break;
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
  EpiParams epi;
};

struct alignas(64) GemmTcParams {
  CUtensorMap wmap[kMaxSeg];   // weight segment maps: box 64 (K) x 128 rows (64 rows when paired)
  CUtensorMap xmap;            // activation map: box 64 (K) x m_tile rows
  EpiParams epi;
  int paired;
  int M;                       // valid activation rows
  int m_tile;                  // activation rows per CTA = MMA N (multiple of 16, <= 256)
  int m_blocks;
  int tmem_cols;
  int num_kb;                  // K / 64
  int splits;                  // K splits = cluster size (1..8)
  int kb_per_split;
  int n_tiles;
  int stages;
  int use_pdl;
};

cudaError_t launch_gemm_simt(const GemmSimtParams& p, int n_tiles, cudaStream_t st, bool pdl);
// Clusters of `splits` CTAs of this GEMM configuration that fit on the GPU at once.
int gemm_tc_max_active_clusters(int m_tile, int stages, int splits);
cudaError_t launch_gemm_tc(const GemmTcParams& p, cudaStream_t st);
size_t gemm_tc_smem_bytes(int m_tile, int stages);
constexpr int kMaxClusterSplits = 8;

}  // namespace dfl
