// Host side of the C ABI (include/dflash.h): validation, workspace, TMA
// descriptors, GEMM planning and the launch sequence of inject / draft.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <map>
#include <tuple>
#include <vector>

#include "../../include/dflash.h"
#include "gemm.cuh"
#include "trace.h"
#include "kernels.cuh"

using namespace dfl;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kAttnTargetCtas = 296;                   // 2 CTAs per SM on 148 SMs
constexpr int kAttnTilesPerCta = 8;                    // longest key-tile chain per attention CTA
constexpr int kAttnAdaptivePairs = 64;                 // (request, KV head) pairs from which the device picks the split size

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// GEMM call sites (profiling tags)
enum GemmTag { TAG_FC = 0, TAG_KV, TAG_QKV, TAG_O, TAG_GATEUP, TAG_DOWN, TAG_LM, TAG_COUNT };
enum ProfKind {
  PK_GEMM_TC = 0,                    // + tag
  PK_GEMM_SIMT = PK_GEMM_TC + TAG_COUNT,   // + tag
  PK_ATTN = PK_GEMM_SIMT + TAG_COUNT,
  PK_ATTN_MERGE,
  PK_EMBED_NORM,
  PK_RMSNORM,
  PK_ARGMAX,
  PK_COPY,
  PK_COUNT
};
const char* const kProfNames[PK_COUNT] = {
    "gemm_tc:fc", "gemm_tc:kv", "gemm_tc:qkv", "gemm_tc:o", "gemm_tc:gateup", "gemm_tc:down", "gemm_tc:lm",
    "gemm_simt:fc", "gemm_simt:kv", "gemm_simt:qkv", "gemm_simt:o", "gemm_simt:gateup", "gemm_simt:down",
    "gemm_simt:lm", "attention", "attention_merge", "embed_norm", "rmsnorm", "argmax_finalize", "hidden_copy"};

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double bytes, flops;
};

}  // namespace

struct dflash_ctx {
  dflash_config cfg;
  bool bf16 = false;
  bool force_simt = false;
  bool cache_f16 = false;   // KV cache pools hold fp16 (bf16 drafter only)
  bool use_pdl = false;
  bool debug = false;
  int force_splits = 0;   // DFLASH_SPLITS: fixed K-split count (experiments)
  int force_stages = 0;   // DFLASH_STAGES: fixed ring depth (experiments)
  int split_slots = 2;    // CTAs per SM the K-split plan fills (DFLASH_SPLIT_SLOTS, experiments)
  unsigned test_stall_ns = 0;   // DFLASH_TEST_STALL_NS: failure-injection hook of the tensor-core GEMM
  bool attn_mma = false;        // DFLASH_ATTN=mma: the mma.sync attention kernel even where tcgen05 applies
  int attn_form = -1;           // DFLASH_ATTN_FORM=full|compact: force the tcgen05 attention form (experiments)
  int attn_l2promo = 3;         // DFLASH_ATTN_L2PROMO=0..3: L2 promotion of the attention's tensor maps (experiments)
  int attn_stages = 5;          // K/V ring depth of the tcgen05 attention (DFLASH_ATTN_STAGES, experiments)
  int attn_plan = -1;           // DFLASH_ATTN_PLAN=host|device: force the host's or the device-side split plan
  int* attn_kps = nullptr;      // the device-side split size of the current draft call
  // GEMM sites (bit 1 kv, 2 qkv, 3 o, 4 gate/up, 5 down) that read their activations
  // as one bf16 plane from single_plane_rows rows on (DFLASH_SINGLE_PLANE=mask,rows)
  unsigned single_plane_mask = 0;
  int single_plane_rows = 1 << 30;
  std::map<std::tuple<int, int, int, int>, int> attn_cluster_cap;   // resident clusters per (d, stages, n, rows)
  int num_sms = 148;
  const void* fc = nullptr;
  const void* embed = nullptr;
  const void* lm_head = nullptr;
  const float* final_norm = nullptr;
  std::vector<const float*> attn_norm, mlp_norm;
  std::vector<const void*> wq, wk, wv, wo, wg, wu, wd;
  // workspace
  char* ws = nullptr;
  size_t ws_bytes = 0;
  float* x = nullptr;
  void* h = nullptr;
  void* q = nullptr;
  void* kb = nullptr;
  void* vb = nullptr;
  void* ao = nullptr;
  void* act = nullptr;
  void* c = nullptr;
  unsigned long long* keys = nullptr;
  float* att_o = nullptr;
  float* att_m = nullptr;
  float* att_l = nullptr;
  size_t att_rows = 0;   // capacity in (split, row) pairs
  int* status = nullptr;
  double* inv_freq = nullptr;   // [head_dim/2] RoPE inverse frequencies
  float2* rope_cs = nullptr;    // [rows][head_dim/2] (cos, sin) of the current call's row positions
  float* sumsq[2] = {nullptr, nullptr};   // deferred-norm partial sums of squares [H/128][rows], ping-pong
  EncodeTiledFn encode = nullptr;
  bool prof = false;
  std::vector<ProfRec> recs;
  std::map<std::tuple<const void*, long long, long long, long long, int>, CUtensorMap> maps;
  std::map<std::vector<long long>, CUtensorMap> maps_nd;   // fp16 tensor maps of the attention kernel
};

namespace {

int q_dim(const dflash_config& c) { return c.n_q_heads * c.head_dim; }
int kv_dim(const dflash_config& c) { return c.n_kv_heads * c.head_dim; }
size_t esize(const dflash_ctx* x) { return x->bf16 ? 2 : 4; }

// A failed CUDA call is reported on stderr with the runtime's message, then as DFLASH_ERR_CUDA.
dflash_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return DFLASH_OK;
  std::fprintf(stderr, "dflash: %s: %s\n", where, cudaGetErrorString(e));
  return DFLASH_ERR_CUDA;
}

// Brackets one launch with CUDA events when profiling is on.
struct ProfScope {
  dflash_ctx* ctx;
  cudaStream_t st;
  ProfRec rec{};
  bool on;
  ProfScope(dflash_ctx* c, int kind, cudaStream_t s, double bytes, double flops) : ctx(c), st(s), on(c->prof) {
    if (!on) return;
    rec.kind = kind;
    rec.bytes = bytes;
    rec.flops = flops;
    cudaEventCreate(&rec.a);
    cudaEventCreate(&rec.b);
    cudaEventRecord(rec.a, st);
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(rec.b, st);
    ctx->recs.push_back(rec);
  }
};

bool get_map(dflash_ctx* ctx, const void* ptr, long long rows, long long K, long long ld, int box_rows,
             CUtensorMap* out) {
  auto key = std::make_tuple(ptr, rows, K, ld, box_rows);
  auto it = ctx->maps.find(key);
  if (it != ctx->maps.end()) {
    *out = it->second;
    return true;
  }
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = ctx->encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  if (ctx->maps.size() > 4096) ctx->maps.clear();
  ctx->maps[key] = m;
  *out = m;
  return true;
}

// fp16 tensor map (128-byte swizzle, zero fill out of bounds), rank 2 or 3;
// dims / box in elements (innermost first), strides in bytes of dims 1.. .
bool get_map_f16(dflash_ctx* ctx, const void* ptr, int rank, const long long* dims, const long long* strides,
                 const int* box, CUtensorMap* out) {
  std::vector<long long> key = {(long long)(uintptr_t)ptr, rank};
  for (int i = 0; i < rank; ++i) key.push_back(dims[i]);
  for (int i = 0; i + 1 < rank; ++i) key.push_back(strides[i]);
  for (int i = 0; i < rank; ++i) key.push_back(box[i]);
  auto it = ctx->maps_nd.find(key);
  if (it != ctx->maps_nd.end()) {
    *out = it->second;
    return true;
  }
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = (cuuint64_t)dims[i];
    bx[i] = (cuuint32_t)box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = (cuuint64_t)strides[i];
  CUtensorMap m;
  static const CUtensorMapL2promotion promo[4] = {CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_64B,
                                                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B};
  CUresult r = ctx->encode(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr), d, st, bx,
                           es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo[ctx->attn_l2promo],
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::fprintf(stderr, "dflash: tensor map encode failed (%d)\n", (int)r);
    return false;
  }
  if (ctx->maps_nd.size() > 4096) ctx->maps_nd.clear();
  ctx->maps_nd[key] = m;
  *out = m;
  return true;
}

struct GemmSpec {
  const void* x = nullptr;
  int ldx = 0, M = 0, K = 0;
  int n_seg = 0;
  const void* w[kMaxSeg] = {};
  int seg_rows[kMaxSeg] = {};
  bool paired = false;
  bool x_split = false;   // x holds hi/lo bf16 planes ([2][M][ldx]), tensor-core path only
  int tag = 0;
  EpiParams epi{};
};

enum { SITE_KV = 1, SITE_QKV = 2, SITE_O = 3, SITE_GATEUP = 4, SITE_DOWN = 5 };

// Whether a GEMM site reads its activations as hi/lo planes at `rows` rows.
bool two_planes(const dflash_ctx* ctx, int site, int rows) {
  if (!ctx->bf16) return false;
  return !((ctx->single_plane_mask >> site) & 1u) || rows < ctx->single_plane_rows;
}

// K splits per output tile (= cluster size): the largest count (<= 8) that keeps
// the grid within split_slots CTAs per SM (default two), so every CTA streams
// from the start and a third slot per SM stays free for the next kernel's CTAs
// to start and prefetch their weights (programmatic dependent launch).
int choose_splits(dflash_ctx* ctx, int units, int num_kb, int m_tile) {
  // CTAs of this shape that fit per SM (the ring budgets below: 74 KB up to 32
  // activation rows, 110 KB up to 64, about 220 KB above)
  const int fit = m_tile <= 32 ? 3 : (m_tile <= 64 ? 2 : 1);
  const int slots = std::min(ctx->split_slots, fit) * ctx->num_sms;
  for (int s = kMaxClusterSplits; s >= 2; --s)
    if (num_kb / s >= 2 && units * s <= slots) return s;
  return 1;
}

int pow2_at_least(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

dflash_status run_gemm(dflash_ctx* ctx, GemmSpec g, cudaStream_t st) {
  EpiParams& e = g.epi;
  e.status = ctx->status;
  e.cache_type = ctx->cache_f16 ? OUT_F16 : (ctx->bf16 ? OUT_BF16 : OUT_F32);
  if (!ctx->bf16) e.out_type = OUT_F32;
  int n_tiles = 0;
  if (g.paired) {
    n_tiles = g.seg_rows[0] / (kTileN / 2);
    e.n_seg = 1;
    e.seg_tile_begin[0] = 0;
    e.seg_tile_begin[1] = n_tiles;
  } else {
    e.n_seg = g.n_seg;
    for (int s = 0; s < g.n_seg; ++s) {
      e.seg_tile_begin[s] = n_tiles;
      n_tiles += g.seg_rows[s] / kTileN;
    }
    e.seg_tile_begin[g.n_seg] = n_tiles;
  }
  if (g.M <= 0 || n_tiles <= 0) return DFLASH_OK;
  const double es_ = (double)esize(ctx);
  const double n_out = g.paired ? (double)g.seg_rows[0] : (double)n_tiles * kTileN;
  const double w_rows = (double)n_tiles * kTileN;
  double out_bytes = 0;
  switch (e.kind) {
    case EPI_RESID: out_bytes = 2.0 * g.M * n_out * 4; break;
    case EPI_ARGMAX: out_bytes = (double)g.M * 8; break;
    default: out_bytes = (double)g.M * n_out * es_; break;
  }
  ProfScope prof(ctx, ((!ctx->bf16 || ctx->force_simt) ? PK_GEMM_SIMT : PK_GEMM_TC) + g.tag, st,
                 w_rows * g.K * es_ + (double)g.M * g.K * es_ + out_bytes, 2.0 * g.M * w_rows * g.K);

  if (!ctx->bf16 || ctx->force_simt) {
    GemmSimtParams p{};
    for (int s = 0; s < g.n_seg; ++s) p.w[s] = g.w[s];
    p.paired = g.paired ? 1 : 0;
    p.x = g.x;
    p.ldx = g.ldx;
    p.M = g.M;
    p.K = g.K;
    p.w_bf16 = ctx->bf16 ? 1 : 0;
    p.x_bf16 = ctx->bf16 ? 1 : 0;
    p.x_plane = g.x_split ? (size_t)g.M * g.ldx : 0;
    p.epi = e;
    return cuda_status(launch_gemm_simt(p, n_tiles, st, ctx->use_pdl), "gemm_simt launch");
  }

  GemmTcParams p;
  std::memset(&p, 0, sizeof(p));
  p.epi = e;
  p.paired = g.paired ? 1 : 0;
  p.M = g.M;
  p.x_split = g.x_split ? 1 : 0;
  p.x_plane_rows = g.M;
  p.m_tile = std::min(g.x_split ? 128 : 256, (g.M + 15) / 16 * 16);
  // One plane, 256-row tiles and fewer output tiles than SMs: a K split would not
  // fit (its receive buffer takes the ring), so a few CTAs would stream everything;
  // take 128 rows (the fusion projection at serving bs16 ran on 32 CTAs).
  if (!g.x_split && p.m_tile == 256 && n_tiles * ((g.M + 255) / 256) <= ctx->num_sms) p.m_tile = 128;
  // Few output tiles at 128 rows but more than the SMs at 64: take 64, so that two
  // CTAs share an SM and each one's epilogue runs under the other's MMAs.
  if (p.m_tile == 128 && g.M > 128 && n_tiles * ((g.M + 127) / 128) <= ctx->num_sms &&
      n_tiles * ((g.M + 63) / 64) > ctx->num_sms)
    p.m_tile = 64;
  p.m_blocks = (g.M + p.m_tile - 1) / p.m_tile;
  // accumulator columns: the hi plane's m_tile, then the lo plane's (read 32 at a time)
  p.tmem_cols = std::max(32, pow2_at_least(p.x_split ? p.m_tile + (p.m_tile + 31) / 32 * 32 : p.m_tile));
  p.num_kb = g.K / 64;
  p.n_tiles = n_tiles;
  const int units = n_tiles * p.m_blocks;
  p.splits = ctx->force_splits > 0 ? std::min(ctx->force_splits, std::max(1, p.num_kb / 2))
                                   : choose_splits(ctx, units, p.num_kb, p.m_tile);
  // ring depth: while m_tile <= 32 keep each CTA (ring + receive buffer) within a
  // third of the SM's shared memory, so three CTAs fit; up to 64 rows, or with more
  // unsplit output tiles than SMs, within half, so two CTAs share an SM and one's
  // epilogue runs under the other's MMAs (measured at serving bs32: QKV 100 -> 72,
  // gate/up 228 -> 185, LM head 691 -> 587 us); otherwise (one CTA per SM) use what
  // fits, as a deeper ring is what a lone CTA streams with. The split epilogue
  // reuses the ring for this split's rows (m_tile x 128 fp32) plus one chunk; if
  // that does not fit, use fewer splits.
  const int sb = kTileN * 64 * 2 + (1 + p.x_split) * p.m_tile * 128;
  const bool two_per_sm = p.m_tile <= 64 || (p.splits == 1 && units > ctx->num_sms);
  const size_t budget = p.m_tile <= 32 ? 74 * 1024 : (two_per_sm ? 110 * 1024 : 220 * 1024);
  const size_t chunk_bytes = (size_t)kChunkRows * kChunkLd * 4;
  for (;;) {
    const size_t fixed = gemm_tc_smem_bytes(p.m_tile, p.x_split, 0, p.splits);
    p.stages = budget > fixed ? (int)std::min<size_t>(8, (budget - fixed) / sb) : 0;
    if (ctx->force_stages >= 2 && fixed + (size_t)ctx->force_stages * sb <= 225 * 1024) p.stages = ctx->force_stages;
    const size_t need = (p.splits > 1 ? (size_t)p.m_tile * kTileN * 4 : 0) + chunk_bytes;
    if (p.stages >= 2 && (size_t)p.stages * sb >= need) break;
    if (p.splits == 1) return DFLASH_ERR_UNSUPPORTED;
    p.splits = p.splits > 2 ? p.splits / 2 : 1;
  }
  p.kb_per_split = (p.num_kb + p.splits - 1) / p.splits;
  if (ctx->debug)
    std::fprintf(stderr, "dflash gemm tag=%d M=%d K=%d tiles=%d m_tile=%d stages=%d splits=%d\n", g.tag, g.M, g.K,
                 n_tiles, p.m_tile, p.stages, p.splits);
  p.use_pdl = ctx->use_pdl ? 1 : 0;
  p.test_stall_ns = ctx->test_stall_ns;
  const int box_w = g.paired ? kTileN / 2 : kTileN;
  const int nmaps = g.paired ? 2 : g.n_seg;
  for (int s = 0; s < nmaps; ++s)
    if (!get_map(ctx, g.w[s], g.seg_rows[s], g.K, g.K, box_w, &p.wmap[s])) return DFLASH_ERR_CUDA;
  if (!get_map(ctx, g.x, (long long)(1 + p.x_split) * g.M, g.K, g.ldx, p.m_tile, &p.xmap)) return DFLASH_ERR_CUDA;
  return cuda_status(launch_gemm_tc(p, st), "gemm_tc launch");
}

// The GEMM's input rows are x ⊙ gain; scale its accumulators by the row's rstd
// from the partial sums of squares the previous residual GEMM left in `part`.
void set_deferred_norm(dflash_ctx* ctx, EpiParams& e, const float* part, int rows) {
  e.norm_part = part;
  e.n_part = ctx->cfg.hidden / kTileN;
  e.ld_part = rows;
  e.norm_inv_h = 1.0f / (float)ctx->cfg.hidden;
  e.norm_eps = ctx->cfg.rms_eps;
}

// ---------------------------------------------------------------- the draft pass's GEMMs
// (R = bs * B activation rows; one builder per call site, shared by
// dflash_draft_block and the GEMM-chain instrumentation call)

// RMSNorm -> q, k, v of the block rows, RoPE on q and k at positions ctx_len + i.
GemmSpec spec_qkv(dflash_ctx* ctx, int l, int R, int B, const int* d_ctx_len) {
  const dflash_config& c = ctx->cfg;
  const int QD = q_dim(c), KVD = kv_dim(c);
  GemmSpec qkv;
  qkv.x = ctx->h;
  qkv.x_split = two_planes(ctx, SITE_QKV, R);
  qkv.ldx = c.hidden;
  qkv.M = R;
  qkv.K = c.hidden;
  qkv.n_seg = 3;
  qkv.w[0] = ctx->wq[l];
  qkv.w[1] = ctx->wk[l];
  qkv.w[2] = ctx->wv[l];
  qkv.seg_rows[0] = QD;
  qkv.seg_rows[1] = KVD;
  qkv.seg_rows[2] = KVD;
  qkv.tag = TAG_QKV;
  qkv.epi.kind = EPI_QKV;
  qkv.epi.out_type = OUT_F16;   // the attention kernels run in fp16
  qkv.epi.out[0] = ctx->q;
  qkv.epi.out[1] = ctx->kb;
  qkv.epi.out[2] = ctx->vb;
  qkv.epi.ld_out[0] = QD;
  qkv.epi.ld_out[1] = KVD;
  qkv.epi.ld_out[2] = KVD;
  qkv.epi.rope_mask = 3u;
  qkv.epi.head_dim = c.head_dim;
  qkv.epi.inv_freq = ctx->inv_freq;
  qkv.epi.rope_cs = ctx->rope_cs;   // filled for these rows by the call's embedding kernel
  qkv.epi.rows_per_req = B;
  qkv.epi.pos_base = d_ctx_len;
  if (l > 0) set_deferred_norm(ctx, qkv.epi, ctx->sumsq[1], R);   // rows carry the previous layer's norm
  return qkv;
}

// x += o · Woᵀ; the MLP norm is deferred: x ⊙ gain now, the row scales in the gate/up epilogue.
GemmSpec spec_o(dflash_ctx* ctx, int l, int R) {
  const dflash_config& c = ctx->cfg;
  GemmSpec o;
  o.x = ctx->ao;
  o.x_split = two_planes(ctx, SITE_O, R);
  o.ldx = q_dim(c);
  o.M = R;
  o.K = q_dim(c);
  o.n_seg = 1;
  o.w[0] = ctx->wo[l];
  o.seg_rows[0] = c.hidden;
  o.tag = TAG_O;
  o.epi.kind = EPI_RESID;
  o.epi.x = ctx->x;
  o.epi.ldx = c.hidden;
  o.epi.gamma_next = ctx->mlp_norm[l];
  o.epi.out_type = OUT_BF16X2;
  o.epi.out_plane = (size_t)R * c.hidden;
  o.epi.xg = ctx->h;
  o.epi.sumsq = ctx->sumsq[0];
  o.epi.ld_part = R;
  return o;
}

// act = silu(h · Wgᵀ) ⊙ (h · Wuᵀ), paired gate / up tiles.
GemmSpec spec_gateup(dflash_ctx* ctx, int l, int R) {
  const dflash_config& c = ctx->cfg;
  GemmSpec gu;
  gu.x = ctx->h;
  gu.x_split = two_planes(ctx, SITE_GATEUP, R);
  gu.ldx = c.hidden;
  gu.M = R;
  gu.K = c.hidden;
  gu.n_seg = 2;
  gu.paired = true;
  gu.w[0] = ctx->wg[l];
  gu.w[1] = ctx->wu[l];
  gu.seg_rows[0] = gu.seg_rows[1] = c.intermediate;
  gu.tag = TAG_GATEUP;
  gu.epi.kind = EPI_SWIGLU;
  gu.epi.out_type = OUT_BF16X2;
  gu.epi.out_plane = (size_t)R * c.intermediate;
  gu.epi.out[0] = ctx->act;
  gu.epi.ld_out[0] = c.intermediate;
  set_deferred_norm(ctx, gu.epi, ctx->sumsq[0], R);
  return gu;
}

// x += act · Wdᵀ; the next layer's attention norm (or the final norm) is deferred the same way.
GemmSpec spec_down(dflash_ctx* ctx, int l, int R) {
  const dflash_config& c = ctx->cfg;
  GemmSpec dn;
  dn.x = ctx->act;
  dn.x_split = two_planes(ctx, SITE_DOWN, R);
  dn.ldx = c.intermediate;
  dn.M = R;
  dn.K = c.intermediate;
  dn.n_seg = 1;
  dn.w[0] = ctx->wd[l];
  dn.seg_rows[0] = c.hidden;
  dn.tag = TAG_DOWN;
  dn.epi.kind = EPI_RESID;
  dn.epi.x = ctx->x;
  dn.epi.ldx = c.hidden;
  const bool last = l + 1 == c.n_layers;
  dn.epi.gamma_next = last ? ctx->final_norm : ctx->attn_norm[l + 1];
  dn.epi.out_type = OUT_BF16X2;
  dn.epi.out_plane = (size_t)R * c.hidden;
  dn.epi.xg = ctx->h;
  dn.epi.sumsq = ctx->sumsq[1];
  dn.epi.ld_part = R;
  return dn;
}

// Final norm (deferred) -> shared LM head -> per-row argmax keys; logits are never stored.
GemmSpec spec_lm(dflash_ctx* ctx, int R) {
  const dflash_config& c = ctx->cfg;
  GemmSpec lm;
  lm.x = ctx->h;
  // The LM head only feeds an argmax: above 32 rows it reads the hi plane alone,
  // which halves its MMA work and activation tiles (from 64 rows on, the split
  // makes it tensor- or shared-memory-bound). The hi plane's rounding (2^-9
  // relative) moves a logit by ~2e-3 (std) at these scales, inside the 1e-2
  // top-2 gap the draft tokens are held to; up to 32 rows the lo plane is free.
  lm.x_split = ctx->bf16 && R <= 32;
  lm.ldx = c.hidden;
  lm.M = R;
  lm.K = c.hidden;
  lm.n_seg = 1;
  lm.w[0] = ctx->lm_head;
  lm.seg_rows[0] = c.vocab;
  lm.tag = TAG_LM;
  lm.epi.kind = EPI_ARGMAX;
  lm.epi.keys = ctx->keys;
  if (c.n_layers > 0) set_deferred_norm(ctx, lm.epi, ctx->sumsq[1], R);
  return lm;
}

#define DFL_CHECK(call)                       \
  do {                                        \
    dflash_status s_ = (call);                \
    if (s_ != DFLASH_OK) return s_;           \
  } while (0)

}  // namespace

extern "C" const char* dflash_status_string(dflash_status s) {
  switch (s) {
    case DFLASH_OK: return "ok";
    case DFLASH_ERR_ARG: return "invalid argument";
    case DFLASH_ERR_CUDA: return "CUDA call failed";
    case DFLASH_ERR_OOM: return "out of device memory";
    case DFLASH_ERR_TIMEOUT: return "device wait timed out";
    case DFLASH_ERR_DEVICE: return "out-of-range id, page or position on the device";
    case DFLASH_ERR_UNSUPPORTED: return "unsupported shape";
  }
  return "unknown status";
}

extern "C" dflash_status dflash_create(const dflash_config* cfg, const dflash_weights* w, dflash_ctx** out) {
  try {
    if (!cfg || !w || !out) return DFLASH_ERR_ARG;
    *out = nullptr;
    const dflash_config& c = *cfg;
    if (c.hidden <= 0 || c.n_layers < 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim <= 0 ||
        c.intermediate <= 0 || c.vocab <= 1 || c.n_feat_layers <= 0 || c.target_hidden <= 0 || c.max_block <= 0 ||
        c.max_batch <= 0 || c.max_inject_rows < 0 || c.page_size <= 0 || !(c.rope_theta > 0.f) || !(c.rms_eps >= 0.f))
      return DFLASH_ERR_ARG;
    if (c.mask_token_id < 0 || c.mask_token_id >= c.vocab) return DFLASH_ERR_ARG;
    if (c.window < 0) return DFLASH_ERR_ARG;
    if (c.n_q_heads % c.n_kv_heads) return DFLASH_ERR_ARG;
    if (c.dtype != DFLASH_F32 && c.dtype != DFLASH_BF16) return DFLASH_ERR_ARG;
    if (c.cache_dtype == DFLASH_F16 && c.dtype != DFLASH_BF16) return DFLASH_ERR_ARG;
    if (!w->fc || !w->embed || !w->lm_head || !w->final_norm) return DFLASH_ERR_ARG;
    if (c.n_layers > 0 && (!w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo || !w->mlp_norm || !w->wgate ||
                           !w->wup || !w->wdown))
      return DFLASH_ERR_ARG;
    // shape support: 128-row weight tiles aligned to segment starts, paired 64-row gate/up tiles
    const int F = c.n_feat_layers * c.target_hidden;
    const int kalign = c.dtype == DFLASH_BF16 ? 64 : 32;
    if (c.head_dim != 64 && c.head_dim != 128) return DFLASH_ERR_UNSUPPORTED;
    if (c.hidden % 128 || q_dim(c) % 128 || kv_dim(c) % 128 || c.intermediate % 64 || c.vocab % 128)
      return DFLASH_ERR_UNSUPPORTED;
    if (c.hidden % kalign || q_dim(c) % kalign || c.intermediate % kalign || F % kalign) return DFLASH_ERR_UNSUPPORTED;
    if ((c.n_q_heads / c.n_kv_heads) * c.max_block > 128) return DFLASH_ERR_UNSUPPORTED;

    dflash_ctx* ctx = new dflash_ctx();
    ctx->cfg = c;
    ctx->bf16 = c.dtype == DFLASH_BF16;
    ctx->cache_f16 = c.cache_dtype == DFLASH_F16;
    const char* env = std::getenv("DFLASH_FORCE_SIMT");
    ctx->force_simt = env && env[0] == '1';
    env = std::getenv("DFLASH_DEBUG");
    ctx->debug = env && env[0] == '1';
    env = std::getenv("DFLASH_SPLITS");
    ctx->force_splits = env ? std::atoi(env) : 0;
    if (ctx->force_splits > kMaxClusterSplits) ctx->force_splits = kMaxClusterSplits;
    env = std::getenv("DFLASH_SPLIT_SLOTS");
    if (env && std::atoi(env) >= 1 && std::atoi(env) <= 3) ctx->split_slots = std::atoi(env);
    env = std::getenv("DFLASH_STAGES");
    ctx->force_stages = env ? std::atoi(env) : 0;
    if (ctx->force_stages > 8) ctx->force_stages = 8;
    env = std::getenv("DFLASH_PDL");
    ctx->use_pdl = !(env && env[0] == '0');
    env = std::getenv("DFLASH_ATTN");
    ctx->attn_mma = env && std::strcmp(env, "mma") == 0;
    env = std::getenv("DFLASH_ATTN_FORM");
    if (env) ctx->attn_form = std::strcmp(env, "compact") == 0 ? 1 : (std::strcmp(env, "full") == 0 ? 0 : -1);
    env = std::getenv("DFLASH_ATTN_L2PROMO");
    if (env && std::atoi(env) >= 0 && std::atoi(env) <= 3) ctx->attn_l2promo = std::atoi(env);
    env = std::getenv("DFLASH_SINGLE_PLANE");
    if (env) {
      unsigned mask = 0;
      int rows = 0;
      if (std::sscanf(env, "%u,%d", &mask, &rows) == 2 && rows >= 0) {
        ctx->single_plane_mask = mask;
        ctx->single_plane_rows = rows;
      }
    }
    env = std::getenv("DFLASH_ATTN_PLAN");
    if (env) ctx->attn_plan = std::strcmp(env, "device") == 0 ? 1 : (std::strcmp(env, "host") == 0 ? 0 : -1);
    env = std::getenv("DFLASH_ATTN_STAGES");
    if (env && std::atoi(env) >= 2 && std::atoi(env) <= kMaxAttnTcStages) ctx->attn_stages = std::atoi(env);
    if (c.head_dim == 128 && ctx->attn_stages > 5) ctx->attn_stages = 5;   // what fits beside Q and P
    // Failure injection (tests only): every tensor-core GEMM epilogue gives up on a
    // barrier nothing arrives at after this many ns (capped at 100 ms), so the
    // call completes with DFLASH_ERR_TIMEOUT and no copy or MMA in flight.
    env = std::getenv("DFLASH_TEST_STALL_NS");
    if (env) {
      const long long v = std::atoll(env);
      ctx->test_stall_ns = v <= 0 ? 0u : (unsigned)std::min(v, 100000000LL);
    }
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev);
    ctx->fc = w->fc;
    ctx->embed = w->embed;
    ctx->lm_head = w->lm_head;
    ctx->final_norm = w->final_norm;
    for (int l = 0; l < c.n_layers; ++l) {
      if (!w->attn_norm[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->mlp_norm[l] || !w->wgate[l] ||
          !w->wup[l] || !w->wdown[l]) {
        delete ctx;
        return DFLASH_ERR_ARG;
      }
      ctx->attn_norm.push_back(w->attn_norm[l]);
      ctx->mlp_norm.push_back(w->mlp_norm[l]);
      ctx->wq.push_back(w->wq[l]);
      ctx->wk.push_back(w->wk[l]);
      ctx->wv.push_back(w->wv[l]);
      ctx->wo.push_back(w->wo[l]);
      ctx->wg.push_back(w->wgate[l]);
      ctx->wu.push_back(w->wup[l]);
      ctx->wd.push_back(w->wdown[l]);
    }

    cudaDriverEntryPointQueryResult qres;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || !fn) {
      delete ctx;
      return DFLASH_ERR_CUDA;
    }
    ctx->encode = reinterpret_cast<EncodeTiledFn>(fn);

    // workspace layout
    const size_t R = (size_t)c.max_batch * c.max_block;
    const size_t Rin = std::max(1, c.max_inject_rows);
    const size_t es = esize(ctx);
    const int g = c.n_q_heads / c.n_kv_heads;
    const size_t nr = (size_t)g * c.max_block;
    ctx->att_rows = ((size_t)kAttnTargetCtas + (size_t)c.max_batch * c.n_kv_heads + 8) * nr;
    // the device-side plan's grid: up to 8 waves of two CTAs per SM
    if ((size_t)c.max_batch * c.n_kv_heads >= (size_t)kAttnAdaptivePairs)
      ctx->att_rows = std::max(ctx->att_rows, (size_t)16 * ctx->num_sms * nr);
    size_t off = 0;
    auto take = [&](size_t bytes) {
      size_t o = off;
      off += align256(bytes);
      return o;
    };
    const size_t o_x = take(R * c.hidden * 4);
    const size_t planes = ctx->bf16 ? 2 : 1;   // bf16 activations are stored as hi/lo planes
    const size_t o_h = take(planes * R * c.hidden * es);
    const size_t o_q = take(R * q_dim(c) * es);
    const size_t o_kb = take(R * kv_dim(c) * es);
    const size_t o_vb = take(R * kv_dim(c) * es);
    const size_t o_ao = take(planes * R * q_dim(c) * es);
    const size_t o_act = take(planes * R * c.intermediate * es);
    const size_t o_c = take(planes * Rin * c.hidden * es);
    const size_t o_keys = take(R * 8);
    const size_t o_atto = take(ctx->att_rows * c.head_dim * 4);
    const size_t o_attm = take(ctx->att_rows * 4);
    const size_t o_attl = take(ctx->att_rows * 4);
    const size_t o_st = take(256);
    const size_t o_kps = take(256);
    const size_t o_freq = take((size_t)c.head_dim / 2 * sizeof(double));
    const size_t o_rope = take(std::max(R, Rin) * (size_t)(c.head_dim / 2) * sizeof(float2));
    const size_t o_ss0 = take((size_t)(c.hidden / 128) * R * 4);
    const size_t o_ss1 = take((size_t)(c.hidden / 128) * R * 4);
    ctx->ws_bytes = off;
    if (cudaMalloc(&ctx->ws, off) != cudaSuccess) {
      cudaGetLastError();
      delete ctx;
      return DFLASH_ERR_OOM;
    }
    if (cudaMemset(ctx->ws, 0, off) != cudaSuccess) {
      cudaFree(ctx->ws);
      delete ctx;
      return DFLASH_ERR_CUDA;
    }
    char* b = ctx->ws;
    ctx->x = (float*)(b + o_x);
    ctx->h = b + o_h;
    ctx->q = b + o_q;
    ctx->kb = b + o_kb;
    ctx->vb = b + o_vb;
    ctx->ao = b + o_ao;
    ctx->act = b + o_act;
    ctx->c = b + o_c;
    ctx->keys = (unsigned long long*)(b + o_keys);
    ctx->att_o = (float*)(b + o_atto);
    ctx->att_m = (float*)(b + o_attm);
    ctx->att_l = (float*)(b + o_attl);
    ctx->status = (int*)(b + o_st);
    ctx->attn_kps = (int*)(b + o_kps);
    ctx->inv_freq = (double*)(b + o_freq);
    ctx->rope_cs = (float2*)(b + o_rope);
    ctx->sumsq[0] = (float*)(b + o_ss0);
    ctx->sumsq[1] = (float*)(b + o_ss1);
    {
      // theta^(-2i/d), i = 0..d/2-1, in double
      std::vector<double> f(c.head_dim / 2);
      for (int i = 0; i < c.head_dim / 2; ++i) f[i] = std::pow((double)c.rope_theta, -2.0 * i / c.head_dim);
      if (cudaMemcpy(ctx->inv_freq, f.data(), f.size() * sizeof(double), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(ctx->ws);
        delete ctx;
        return DFLASH_ERR_CUDA;
      }
    }
    *out = ctx;
    return DFLASH_OK;
  } catch (...) {   // no C++ exception crosses the C ABI
    return DFLASH_ERR_OOM;
  }
}

extern "C" void dflash_destroy(dflash_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  cudaFree(ctx->ws);
  delete ctx;
}

extern "C" dflash_status dflash_profile_enable(dflash_ctx* ctx, int enable) {
  if (!ctx) return DFLASH_ERR_ARG;
  ctx->prof = enable != 0;
  return DFLASH_OK;
}

extern "C" int dflash_profile_read(dflash_ctx* ctx, dflash_profile_entry* out, int max_entries) {
  try {
    if (!ctx || (!out && max_entries > 0)) return -(int)DFLASH_ERR_ARG;
    dflash_profile_entry agg[PK_COUNT];
    std::memset(agg, 0, sizeof(agg));
    bool fail = false;
    for (ProfRec& r : ctx->recs) {
      float ms = 0.f;
      if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) fail = true;
      agg[r.kind].launches += 1;
      agg[r.kind].total_ms += ms;
      agg[r.kind].bytes += r.bytes;
      agg[r.kind].flops += r.flops;
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    ctx->recs.clear();
    if (fail) return -(int)DFLASH_ERR_CUDA;
    int n = 0;
    for (int k = 0; k < PK_COUNT; ++k) {
      if (!agg[k].launches) continue;
      if (n < max_entries) {
        out[n] = agg[k];
        std::strncpy(out[n].name, kProfNames[k], sizeof(out[n].name) - 1);
      }
      ++n;
    }
    return std::min(n, max_entries);
  } catch (...) {   // no C++ exception crosses the C ABI
    return -1;
  }
}

extern "C" dflash_status dflash_get_error(dflash_ctx* ctx, void* stream) {
  if (!ctx) return DFLASH_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DFLASH_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ctx->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DFLASH_ERR_CUDA;
  if (v && cudaMemset(ctx->status, 0, sizeof(int)) != cudaSuccess) return DFLASH_ERR_CUDA;
  if (v & ST_TIMEOUT) return DFLASH_ERR_TIMEOUT;
  if (v) return DFLASH_ERR_DEVICE;
  return DFLASH_OK;
}

extern "C" dflash_status dflash_inject_ctx(dflash_ctx* ctx, const void* feats, int bs, int max_new,
                                           const int* d_n_new, const int* d_start_pos, void* const* k_cache,
                                           void* const* v_cache, const int* d_page_table, int max_pages,
                                           int num_pages, void* stream) {
  dfl::TraceRange trace_("dflash_inject_ctx");
  try {
    if (!ctx) return DFLASH_ERR_ARG;
    const dflash_config& c = ctx->cfg;
    if (bs <= 0 || bs > c.max_batch || max_new < 0 || (long long)bs * max_new > c.max_inject_rows)
      return DFLASH_ERR_ARG;
    if (max_new == 0) return DFLASH_OK;
    if (!feats || !d_n_new || !d_start_pos || !d_page_table || max_pages <= 0 || num_pages <= 0) return DFLASH_ERR_ARG;
    if (c.n_layers > 0 && (!k_cache || !v_cache)) return DFLASH_ERR_ARG;
    for (int l = 0; l < c.n_layers; ++l)
      if (!k_cache[l] || !v_cache[l]) return DFLASH_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int M = bs * max_new;
    const int F = c.n_feat_layers * c.target_hidden;

    GemmSpec fcg;
    fcg.x = feats;
    fcg.ldx = F;
    fcg.M = M;
    fcg.K = F;
    fcg.n_seg = 1;
    fcg.w[0] = ctx->fc;
    fcg.seg_rows[0] = c.hidden;
    fcg.tag = TAG_FC;
    fcg.epi.kind = EPI_STORE;
    fcg.epi.out[0] = ctx->c;
    fcg.epi.ld_out[0] = c.hidden;
    fcg.epi.out_type = OUT_BF16X2;   // c feeds the K/V GEMM as hi/lo planes
    fcg.epi.out_plane = (size_t)M * c.hidden;
    fcg.epi.rows_per_req = max_new;
    // side job of the fusion GEMM: the RoPE table of the injected rows' positions
    fcg.epi.fill = RopeFill{d_start_pos, max_new, M, c.head_dim / 2, ctx->inv_freq, ctx->rope_cs};
    DFL_CHECK(run_gemm(ctx, fcg, st));

    // all layers' K and V projections of c, up to kMaxSeg segments per launch
    const int per_launch = kMaxSeg / 2;
    for (int l0 = 0, part = 0; l0 < c.n_layers; l0 += per_launch, ++part) {
      const int nl = std::min(per_launch, c.n_layers - l0);
      GemmSpec kv;
      kv.x = ctx->c;
      kv.x_split = two_planes(ctx, SITE_KV, M);
      kv.ldx = c.hidden;
      kv.M = M;
      kv.K = c.hidden;
      kv.n_seg = 2 * nl;
      kv.tag = TAG_KV;
      EpiParams& e = kv.epi;
      e.kind = EPI_KV_INJECT;
      for (int i = 0; i < nl; ++i) {
        kv.w[2 * i] = ctx->wk[l0 + i];
        kv.w[2 * i + 1] = ctx->wv[l0 + i];
        kv.seg_rows[2 * i] = kv.seg_rows[2 * i + 1] = kv_dim(c);
        e.out[2 * i] = k_cache[l0 + i];
        e.out[2 * i + 1] = v_cache[l0 + i];
        e.rope_mask |= 1u << (2 * i);
      }
      e.head_dim = c.head_dim;
      e.inv_freq = ctx->inv_freq;
      e.rope_cs = ctx->rope_cs;
      e.rows_per_req = max_new;
      e.pos_base = d_start_pos;
      e.row_count = d_n_new;
      e.page_table = d_page_table;
      e.max_pages = max_pages;
      e.num_pages = num_pages;
      e.page_size = c.page_size;
      e.n_kv = c.n_kv_heads;
      DFL_CHECK(run_gemm(ctx, kv, st));
    }
    return DFLASH_OK;
  } catch (...) {   // no C++ exception crosses the C ABI
    return DFLASH_ERR_OOM;
  }
}

namespace {

// Sampled drafting (temperature > 0): the LM head draws each draft token by the
// Gumbel-max rule and stores the drafter's logits for the sampled verify.
struct SampleArgs {
  float inv_temp;
  uint32_t seed_lo, seed_hi;
  float* logits_out;
};

dflash_status draft_impl(dflash_ctx* ctx, const int* d_anchor, const int* d_ctx_len, int bs, int B,
                         const void* const* k_cache, const void* const* v_cache, const int* d_page_table,
                         int max_pages, int num_pages, int max_ctx, int* d_draft, float* d_hidden_out, void* stream,
                         const SampleArgs* smp) {
  try {
    if (!ctx) return DFLASH_ERR_ARG;
    const dflash_config& c = ctx->cfg;
    if (bs <= 0 || bs > c.max_batch || B <= 0 || B > c.max_block || max_ctx < 0) return DFLASH_ERR_ARG;
    if (!d_anchor || !d_ctx_len || (B > 1 && !d_draft)) return DFLASH_ERR_ARG;
    if (c.n_layers > 0 && (!k_cache || !v_cache)) return DFLASH_ERR_ARG;
    for (int l = 0; l < c.n_layers; ++l)
      if (!k_cache[l] || !v_cache[l]) return DFLASH_ERR_ARG;
    if (max_ctx > 0 && (!d_page_table || max_pages <= 0 || num_pages <= 0)) return DFLASH_ERR_ARG;
    if (max_ctx > (long long)max_pages * c.page_size) return DFLASH_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int R = bs * B;
    const int H = c.hidden, QD = q_dim(c), KVD = kv_dim(c);
    const int hb = ctx->bf16 ? 1 : 0;
    const size_t layer_stride = (size_t)R * H;

    const double es = (double)esize(ctx);
    const double norm_bytes = (double)R * H * (4 + es);

    // attention split plan. The context of the longest request is cut into n_splits
    // ranges of kps keys (a multiple of the kernel's key tile); the last range also
    // takes the B block keys. Tensor-core path: the splits of one (request, KV head)
    // form a cluster (<= 16) and merge through distributed shared memory. With few
    // (request, KV head) pairs and <= 64 query rows the kernel runs two key groups
    // per CTA and one wave of CTAs (one per SM); otherwise one key group and about
    // two CTAs per SM. Long contexts get enough splits for <= kAttnTilesPerCta key
    // tiles per CTA; when 16 splits leave both the GPU under-filled and the CTAs
    // long, the splits write their partials to global memory and a second kernel
    // merges them (any split count).
    const int g = c.n_q_heads / c.n_kv_heads;
    const int pairs = bs * c.n_kv_heads;
    const int key_tile = ctx->bf16 ? 64 : 32;
    // keys a request's block can attend to: the whole context, or with a sliding
    // window at most window + 63 from the window's 64-aligned start
    const int span = c.window > 0 ? std::min(max_ctx, c.window + 63) : max_ctx;
    const int ctx_tiles = std::max(1, (span + key_tile - 1) / key_tile);
    int attn_ks = 1, n_splits;
    bool attn_gmerge = false;
    if (ctx->bf16) {
      const bool small = g * B <= 64 && ctx->num_sms / pairs >= 8;
      const int want = small ? ctx->num_sms / pairs : (kAttnTargetCtas + pairs - 1) / pairs;
      n_splits = std::min(want, kMaxAttnCluster);
      attn_ks = 2;   // two key groups per CTA (two CTAs per SM at <= 64 query rows, one at 128)
      if ((ctx_tiles + n_splits - 1) / n_splits > kAttnTilesPerCta && pairs * kMaxAttnCluster < kAttnTargetCtas) {
        // long context, few pairs: one wave of two-group CTAs (one per SM at 128
        // query rows, two at <= 64), partials merged by a second kernel
        attn_gmerge = true;
        const int per_sm = g * B > 64 ? 1 : 2;
        n_splits = std::min(ctx_tiles, std::max(n_splits, (per_sm * ctx->num_sms + pairs - 1) / pairs));
      }
    } else {
      n_splits = std::max(1, (kAttnTargetCtas + pairs - 1) / pairs);
    }
    int kps = (std::max(span, 1) + n_splits - 1) / n_splits;
    kps = (kps + key_tile - 1) / key_tile * key_tile;
    n_splits = std::max(1, (span + kps - 1) / kps);
    // Tensor-core (tcgen05) attention: bf16 drafter, fp16 cache, 64-key tiles that
    // stay inside one page. Two forms: full (one CTA per SM, a ring of
    // attn_stages K/V tiles) and compact (two CTAs per SM, two stages each). For
    // the chosen form the split count minimises waves x CTA time, a CTA's time in
    // units of one key tile being a start-up (first HBM round trip, merge) plus
    // its tiles (the rate a lone CTA sustains is set by its S -> softmax -> P·V
    // chain, not by HBM),
    // where the clusters resident per wave come from the occupancy query (a
    // cluster merges through distributed shared memory, at most 16 CTAs), or uses
    // one wave of CTAs with a global merge (a second kernel) and any split count.
    const bool attn_tc = ctx->bf16 && ctx->cache_f16 && !ctx->attn_mma && c.page_size % 64 == 0 && g * B <= 128 &&
                         (c.head_dim == 64 || c.head_dim == 128);
    bool attn_compact = false;
    AttnKpsPlan kplan{};   // out == null: the host's split size
    if (attn_tc) {
      const int nr = g * B;
      const int blk_tiles = (B + 63) / 64;
      // Form: with few (request, KV head) pairs the full form's deeper pipeline wins;
      // from 16 pairs on, two CTAs per SM hide each other's per-tile chain (both
      // measured on B200 across the benchmark workloads).
      const int want_form = ctx->attn_form >= 0 ? ctx->attn_form : (pairs >= 16 ? 1 : 0);
      constexpr double kStart = 4.0, kMergeKernel = 3.0;
      double best = 1e30;
      for (int form = 0; form < 2; ++form) {
        const bool compact = form == 1;
        if (form != want_form) continue;
        const int st_n = compact ? 2 : ctx->attn_stages;
        const double t_tile = compact ? 1.25 : 1.0;
        for (int sp = 1; sp <= kMaxAttnCluster; ++sp) {
          int kp = (std::max(span, 1) + sp - 1) / sp;
          kp = (kp + 63) / 64 * 64;
          if (std::max(1, (span + kp - 1) / kp) != sp) continue;
          auto key = std::make_tuple(c.head_dim * 2 + (int)compact, st_n, sp, nr);
          auto it = ctx->attn_cluster_cap.find(key);
          const int cap =
              it != ctx->attn_cluster_cap.end()
                  ? it->second
                  : (ctx->attn_cluster_cap[key] = attn_tc_max_clusters(c.head_dim, compact, st_n, sp, false, nr));
          if (ctx->debug && sp <= 4) std::fprintf(stderr, "dflash attention form %d cluster %d: %d resident\n", form, sp, cap);
          if (cap < 1) continue;
          const double cost = (double)((pairs + cap - 1) / cap) * (kStart + (kp / 64 + blk_tiles) * t_tile);
          if (cost < best) {
            best = cost;
            n_splits = sp;
            kps = kp;
            attn_gmerge = false;
            attn_compact = compact;
          }
        }
        // global merge: every CTA resident at once, any split count
        const int per_sm = compact ? 2 : 1;
        const int sp_max =
            std::min(per_sm * ctx->num_sms / std::max(pairs, 1), (int)(ctx->att_rows / ((size_t)pairs * nr)));
        for (int sp = 2; sp <= sp_max; ++sp) {
          int kp = (std::max(span, 1) + sp - 1) / sp;
          kp = (kp + 63) / 64 * 64;
          if (std::max(1, (span + kp - 1) / kp) != sp) continue;
          const double cost = kStart + kMergeKernel + (kp / 64 + blk_tiles) * t_tile;
          if (cost < best) {
            best = cost;
            n_splits = sp;
            kps = kp;
            attn_gmerge = true;
            attn_compact = compact;
          }
        }
      }
      if (best >= 1e30) return DFLASH_ERR_UNSUPPORTED;
      // A global merge chosen in the full form (long contexts, few pairs): run it in
      // the compact form, two CTAs per SM with half the keys each (measured at the
      // Coder-30B shape, bs 1: B 16 1340 -> 1365, B 8 1428 -> 1487 cycles/s).
      if (ctx->attn_form < 0 && attn_gmerge && !attn_compact) {
        const int sp_max = std::min(2 * ctx->num_sms / std::max(pairs, 1), (int)(ctx->att_rows / ((size_t)pairs * nr)));
        double best_c = 1e30;
        for (int sp = 2; sp <= sp_max; ++sp) {
          int kp = (std::max(span, 1) + sp - 1) / sp;
          kp = (kp + 63) / 64 * 64;
          if (std::max(1, (span + kp - 1) / kp) != sp) continue;
          const double cost = kStart + kMergeKernel + (kp / 64 + blk_tiles) * 1.25;
          if (cost < best_c) {
            best_c = cost;
            n_splits = sp;
            kps = kp;
            attn_compact = true;
          }
        }
      }
      // Many (request, KV head) pairs: the batch's contexts are usually ragged, and
      // a plan for the longest request leaves most CTA slots idle behind it. The
      // global merge then takes a split size that the device picks from the actual
      // context lengths (the embedding kernel, AttnKpsPlan: fewest waves x CTA
      // time). The flat grid covers the smallest split size allowed, items in
      // order; CTAs past the batch's items come last and exit at once.
      const bool adaptive = ctx->attn_plan == 1 || (ctx->attn_plan < 0 && pairs >= kAttnAdaptivePairs);
      if (adaptive) {
        const int slots = (want_form == 1 ? 2 : 1) * ctx->num_sms;
        const int keys = span + B;   // a request's keys: its (window of) context and the block
        const int key_tiles = (keys + 63) / 64;
        int min_tiles =
            std::max(4, (int)(((long long)pairs * key_tiles + 8LL * slots - 1) / (8LL * slots)));   // grid <= 8 waves
        int sp = (keys + 64 * min_tiles - 1) / (64 * min_tiles);
        while ((size_t)pairs * sp * nr > ctx->att_rows && sp > 1) {
          ++min_tiles;
          sp = (keys + 64 * min_tiles - 1) / (64 * min_tiles);
        }
        if ((size_t)pairs * sp * nr <= ctx->att_rows) {
          kplan = AttnKpsPlan{d_ctx_len, bs, B, c.window, max_ctx, min_tiles, slots, c.n_kv_heads, ctx->attn_kps};
          n_splits = std::max(1, sp);
          kps = 64 * min_tiles;
          attn_gmerge = true;
          attn_compact = want_form == 1;
        }
      }
    }
    if (ctx->debug)
      std::fprintf(stderr, "dflash attention %s%s pairs=%d splits=%d kps=%d gmerge=%d span=%d%s\n",
                   attn_tc ? "tcgen05" : (ctx->bf16 ? "mma.sync" : "simt"), attn_compact ? " compact" : "", pairs,
                   n_splits, kps, (int)attn_gmerge, span, kplan.out ? " (split size chosen on the device)" : "");
    // split partials in global memory (CUDA-core path, or the global merge) must fit the workspace
    if ((!ctx->bf16 || attn_gmerge) && (size_t)bs * c.n_kv_heads * n_splits * g * B > ctx->att_rows)
      return DFLASH_ERR_UNSUPPORTED;
    {
      ProfScope prof(ctx, PK_EMBED_NORM, st, (double)R * H * (es + 4 + es), 0);
      // the embedding kernel also fills the RoPE table of the block rows' positions
      // (and, for the device-side attention plan, the call's split size)
      const RopeFill rf{d_ctx_len, B, R, c.head_dim / 2, ctx->inv_freq, ctx->rope_cs};
      DFL_CHECK(cuda_status(launch_embed_norm(ctx->embed, hb, d_anchor, c.mask_token_id, nullptr, nullptr, B, R,
                                              c.vocab, H,
                                              c.n_layers > 0 ? ctx->attn_norm[0] : ctx->final_norm, c.rms_eps,
                                              ctx->x, ctx->h, hb, hb ? (size_t)R * H : 0, ctx->status, rf, kplan, st,
                                              ctx->use_pdl),
                            "embed_norm launch"));
    }

    for (int l = 0; l < c.n_layers; ++l) {
      DFL_CHECK(run_gemm(ctx, spec_qkv(ctx, l, R, B, d_ctx_len), st));

      AttnParams ap{};
      ap.q = ctx->q;
      ap.kblk = ctx->kb;
      ap.vblk = ctx->vb;
      ap.kc = k_cache[l];
      ap.vc = v_cache[l];
      ap.ctx_len = d_ctx_len;
      ap.page_table = d_page_table;
      ap.max_pages = max_pages;
      ap.num_pages = num_pages;
      ap.page_size = c.page_size;
      ap.bs = bs;
      ap.B = B;
      ap.n_q = c.n_q_heads;
      ap.n_kv = c.n_kv_heads;
      ap.d = c.head_dim;
      ap.g = g;
      ap.kps = kps;
      ap.n_splits = n_splits;
      ap.ks = attn_ks;
      ap.global_merge = attn_gmerge ? 1 : 0;
      ap.kps_dev = kplan.out;
      ap.max_ctx = max_ctx;
      ap.window = c.window;
      ap.scale = (float)(1.0 / std::sqrt((double)c.head_dim));
      ap.part_o = ctx->att_o;
      ap.part_m = ctx->att_m;
      ap.part_l = ctx->att_l;
      ap.status = ctx->status;
      ap.out_plane = (size_t)R * QD;
      ap.cache_f16 = ctx->cache_f16 ? 1 : 0;
      {
        // context K/V of every request (upper bound max_ctx), block q/k/v, output
        const double kvb = (double)bs * span * KVD * 2 * es + (double)R * (2 * QD + 2 * KVD) * es;
        const double fl = 4.0 * bs * B * (double)(span + B) * QD;
        ProfScope prof(ctx, PK_ATTN, st, kvb, fl);
        if (attn_tc) {
          AttnTcParams tp;
          std::memset(&tp, 0, sizeof(tp));
          tp.a = ap;
          tp.stages = ctx->attn_stages;
          tp.compact = attn_compact ? 1 : 0;
          const int D = c.head_dim;
          const long long qd[3] = {D, c.n_q_heads, R}, qs[2] = {(long long)D * 2, (long long)QD * 2};
          const int qb[3] = {64, g, B};
          const long long bd[3] = {KVD, B, bs}, bst[2] = {(long long)KVD * 2, (long long)B * KVD * 2};
          const int bb[3] = {64, 64, 1};
          const long long cd[2] = {D, (long long)num_pages * c.n_kv_heads * c.page_size}, cst[1] = {(long long)D * 2};
          const int cb[2] = {64, 64};
          if (!get_map_f16(ctx, ctx->q, 3, qd, qs, qb, &tp.qmap) || !get_map_f16(ctx, ctx->kb, 3, bd, bst, bb, &tp.kbmap) ||
              !get_map_f16(ctx, ctx->vb, 3, bd, bst, bb, &tp.vbmap) ||
              !get_map_f16(ctx, k_cache[l], 2, cd, cst, cb, &tp.kcmap) ||
              !get_map_f16(ctx, v_cache[l], 2, cd, cst, cb, &tp.vcmap))
            return DFLASH_ERR_CUDA;
          DFL_CHECK(cuda_status(launch_attn_tc(tp, ctx->ao, st, ctx->use_pdl), "attention (tcgen05) launch"));
        } else {
          DFL_CHECK(cuda_status(launch_attention(ap, ctx->ao, hb, hb, st, ctx->use_pdl), "attention launch"));
        }
      }
      if (attn_tc && attn_gmerge) {
        // partials: n_splits x (O, m, l) per query row, read once; the output rows (two planes)
        const double pb = (double)bs * c.n_kv_heads * n_splits * g * B * (c.head_dim + 2) * 4 + (double)R * QD * 2 * es;
        ProfScope prof2(ctx, PK_ATTN_MERGE, st, pb, 0);
        DFL_CHECK(cuda_status(launch_attn_gmerge(ap, ctx->ao, st, ctx->use_pdl), "attention merge launch"));
      }

      DFL_CHECK(run_gemm(ctx, spec_o(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_gateup(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_down(ctx, l, R), st));
      const bool last = l + 1 == c.n_layers;

      if (d_hidden_out) {
        ProfScope prof(ctx, PK_COPY, st, (double)layer_stride * 8, 0);
        if (cudaMemcpyAsync(d_hidden_out + l * layer_stride, ctx->x, layer_stride * 4, cudaMemcpyDeviceToDevice,
                            st) != cudaSuccess)
          return DFLASH_ERR_CUDA;
        if (last) {
          // the final normed rows, for parity checks only (the LM head uses the deferred form)
          ProfScope prof2(ctx, PK_RMSNORM, st, norm_bytes, 0);
          DFL_CHECK(cuda_status(launch_rmsnorm(ctx->x, R, H, ctx->final_norm, c.rms_eps, nullptr, hb,
                                               d_hidden_out + (size_t)c.n_layers * layer_stride, st, ctx->use_pdl),
                                "rmsnorm launch"));
        }
      }
    }
    if (c.n_layers == 0 && d_hidden_out)
      DFL_CHECK(cuda_status(launch_rmsnorm(ctx->x, R, H, ctx->final_norm, c.rms_eps, ctx->h, hb, d_hidden_out, st,
                                           ctx->use_pdl),
                            "rmsnorm launch"));

    {
      GemmSpec lm = spec_lm(ctx, R);
      if (smp) {
        lm.epi.kind = EPI_SAMPLE;
        lm.epi.inv_temp = smp->inv_temp;
        lm.epi.seed_lo = smp->seed_lo;
        lm.epi.seed_hi = smp->seed_hi;
        lm.epi.logits_out = smp->logits_out;
        lm.epi.ld_logits = c.vocab;
        lm.epi.rows_per_req = B;
      }
      DFL_CHECK(run_gemm(ctx, lm, st));
    }
    {
      ProfScope prof(ctx, PK_ARGMAX, st, (double)R * 8 * 2 + (double)bs * (B - 1) * 4, 0);
      const dflash_status fs = cuda_status(launch_argmax_finalize(ctx->keys, bs, B, d_draft, st, ctx->use_pdl),
                                           "argmax_finalize launch");
      if (fs != DFLASH_OK) {
        // the LM head has folded its maxima into the keys: clear them, or the next
        // draft would start from this call's keys
        cudaMemsetAsync(ctx->keys, 0, (size_t)R * sizeof(unsigned long long), st);
        return fs;
      }
    }
    return DFLASH_OK;
  } catch (...) {   // no C++ exception crosses the C ABI
    return DFLASH_ERR_OOM;
  }
}

}  // namespace

extern "C" dflash_status dflash_draft_block(dflash_ctx* ctx, const int* d_anchor, const int* d_ctx_len, int bs,
                                            int B, const void* const* k_cache, const void* const* v_cache,
                                            const int* d_page_table, int max_pages, int num_pages, int max_ctx,
                                            int* d_draft, float* d_hidden_out, void* stream) {
  dfl::TraceRange trace_("dflash_draft_block");
  return draft_impl(ctx, d_anchor, d_ctx_len, bs, B, k_cache, v_cache, d_page_table, max_pages, num_pages, max_ctx,
                    d_draft, d_hidden_out, stream, nullptr);
}

extern "C" dflash_status dflash_draft_block_sample(dflash_ctx* ctx, const int* d_anchor, const int* d_ctx_len,
                                                   int bs, int B, const void* const* k_cache,
                                                   const void* const* v_cache, const int* d_page_table,
                                                   int max_pages, int num_pages, int max_ctx, float temperature,
                                                   unsigned long long seed, int* d_draft, float* d_draft_logits,
                                                   float* d_hidden_out, void* stream) {
  dfl::TraceRange trace_("dflash_draft_block_sample");
  if (!ctx) return DFLASH_ERR_ARG;
  if (!(temperature > 0.f) || !std::isfinite(temperature)) return DFLASH_ERR_ARG;
  if (B > 1 && !d_draft_logits) return DFLASH_ERR_ARG;
  SampleArgs smp;
  smp.inv_temp = 1.0f / temperature;
  smp.seed_lo = (uint32_t)(seed & 0xffffffffull);
  smp.seed_hi = (uint32_t)(seed >> 32);
  smp.logits_out = d_draft_logits;
  return draft_impl(ctx, d_anchor, d_ctx_len, bs, B, k_cache, v_cache, d_page_table, max_pages, num_pages, max_ctx,
                    d_draft, d_hidden_out, stream, &smp);
}

extern "C" dflash_status dflash_profile_gemm_chain(dflash_ctx* ctx, const void* feats, int bs, int max_new,
                                                   const int* d_n_new, const int* d_start_pos, void* const* k_cache,
                                                   void* const* v_cache, const int* d_page_table, int max_pages,
                                                   int num_pages, const int* d_ctx_len, int B, void* stream) {
  dfl::TraceRange trace_("dflash_profile_gemm_chain");
  try {
    if (!ctx) return DFLASH_ERR_ARG;
    const dflash_config& c = ctx->cfg;
    if (!ctx->bf16 || ctx->force_simt) return DFLASH_ERR_UNSUPPORTED;   // the chain times the tensor-core GEMM
    if (bs <= 0 || bs > c.max_batch || B <= 0 || B > c.max_block || !d_ctx_len) return DFLASH_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the injection is GEMMs only: run it as dflash_inject_ctx does
    DFL_CHECK(dflash_inject_ctx(ctx, feats, bs, max_new, d_n_new, d_start_pos, k_cache, v_cache, d_page_table,
                                max_pages, num_pages, stream));
    const int R = bs * B;
    for (int l = 0; l < c.n_layers; ++l) {
      DFL_CHECK(run_gemm(ctx, spec_qkv(ctx, l, R, B, d_ctx_len), st));
      DFL_CHECK(run_gemm(ctx, spec_o(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_gateup(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_down(ctx, l, R), st));
    }
    DFL_CHECK(run_gemm(ctx, spec_lm(ctx, R), st));
    // the LM head folded its maxima into the keys; the next draft must start from zero
    return cuda_status(cudaMemsetAsync(ctx->keys, 0, (size_t)R * sizeof(unsigned long long), st), "keys reset");
  } catch (...) {   // no C++ exception crosses the C ABI
    return DFLASH_ERR_OOM;
  }
}

extern "C" dflash_status dflash_target_forward(dflash_ctx* ctx, const int* d_tokens, const int* d_anchor,
                                               const int* d_draft, int bs, int n, const int* d_pos0,
                                               void* const* k_cache, void* const* v_cache, const int* d_page_table,
                                               int max_pages, int num_pages, int max_ctx, const int* taps, int n_taps,
                                               float* d_logits, float* d_feats, void* stream) {
  dfl::TraceRange trace_("dflash_target_forward");
  try {
    if (!ctx) return DFLASH_ERR_ARG;
    const dflash_config& c = ctx->cfg;
    if (ctx->bf16) return DFLASH_ERR_UNSUPPORTED;   // the causal path is the fp32 one
    if (bs <= 0 || bs > c.max_batch || n <= 0 || n > c.max_block || max_ctx < 0) return DFLASH_ERR_ARG;
    if (!d_tokens && (!d_anchor || (n > 1 && !d_draft))) return DFLASH_ERR_ARG;
    if (!d_pos0 || !d_page_table || max_pages <= 0 || num_pages <= 0 || !d_logits) return DFLASH_ERR_ARG;
    if (c.n_layers > 0 && (!k_cache || !v_cache)) return DFLASH_ERR_ARG;
    for (int l = 0; l < c.n_layers; ++l)
      if (!k_cache[l] || !v_cache[l]) return DFLASH_ERR_ARG;
    if (n_taps < 0 || (n_taps > 0 && (!taps || !d_feats))) return DFLASH_ERR_ARG;
    for (int f = 0; f < n_taps; ++f)
      if (taps[f] < 0 || taps[f] >= c.n_layers || (f > 0 && taps[f] <= taps[f - 1])) return DFLASH_ERR_ARG;
    if ((long long)max_ctx + n > (long long)max_pages * c.page_size) return DFLASH_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int R = bs * n;
    const int H = c.hidden, KVD = kv_dim(c);

    const RopeFill rf{d_pos0, n, R, c.head_dim / 2, ctx->inv_freq, ctx->rope_cs};
    DFL_CHECK(cuda_status(launch_embed_norm(ctx->embed, 0, d_anchor, c.mask_token_id, d_tokens, d_draft, n, R,
                                            c.vocab, H, c.n_layers > 0 ? ctx->attn_norm[0] : ctx->final_norm,
                                            c.rms_eps, ctx->x, ctx->h, 0, 0, ctx->status, rf, AttnKpsPlan{}, st,
                                            ctx->use_pdl),
                          "embed_norm launch"));
    // The split plan depends on bs and max_ctx only (not on n or the rows' positions),
    // so a row's attention is the same arithmetic in a block forward and in a
    // one-token forward given the same max_ctx.
    const int g = c.n_q_heads / c.n_kv_heads;
    const int pairs = bs * c.n_kv_heads;
    int n_splits = std::max(1, (kAttnTargetCtas + pairs - 1) / pairs);
    int kps = (std::max(max_ctx, 1) + n_splits - 1) / n_splits;
    kps = (kps + 31) / 32 * 32;
    n_splits = std::max(1, (max_ctx + kps - 1) / kps);
    if ((size_t)bs * c.n_kv_heads * n_splits * g * n > ctx->att_rows) return DFLASH_ERR_UNSUPPORTED;

    for (int l = 0; l < c.n_layers; ++l) {
      DFL_CHECK(run_gemm(ctx, spec_qkv(ctx, l, R, n, d_pos0), st));
      // the block's own keys and values join the target's cache (a causal decoder)
      DFL_CHECK(cuda_status(launch_kv_scatter((const float*)ctx->kb, (const float*)ctx->vb, d_pos0, n, R, c.n_kv_heads,
                                              c.head_dim, d_page_table, max_pages, num_pages, c.page_size,
                                              (float*)k_cache[l], (float*)v_cache[l], ctx->status, st),
                            "kv scatter launch"));
      AttnParams ap{};
      ap.q = ctx->q;
      ap.kblk = ctx->kb;
      ap.vblk = ctx->vb;
      ap.kc = k_cache[l];
      ap.vc = v_cache[l];
      ap.ctx_len = d_pos0;   // context: cache positions before the block
      ap.page_table = d_page_table;
      ap.max_pages = max_pages;
      ap.num_pages = num_pages;
      ap.page_size = c.page_size;
      ap.bs = bs;
      ap.B = n;
      ap.n_q = c.n_q_heads;
      ap.n_kv = c.n_kv_heads;
      ap.d = c.head_dim;
      ap.g = g;
      ap.kps = kps;
      ap.n_splits = n_splits;
      ap.ks = 1;
      ap.max_ctx = max_ctx;
      ap.scale = (float)(1.0 / std::sqrt((double)c.head_dim));
      ap.part_o = ctx->att_o;
      ap.part_m = ctx->att_m;
      ap.part_l = ctx->att_l;
      ap.status = ctx->status;
      ap.causal = 1;
      DFL_CHECK(cuda_status(launch_attention(ap, ctx->ao, 0, 0, st, ctx->use_pdl), "attention launch"));
      DFL_CHECK(run_gemm(ctx, spec_o(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_gateup(ctx, l, R), st));
      DFL_CHECK(run_gemm(ctx, spec_down(ctx, l, R), st));
      for (int f = 0; f < n_taps; ++f)
        if (taps[f] == l && cudaMemcpy2DAsync(d_feats + (size_t)f * H, (size_t)n_taps * H * 4, ctx->x, (size_t)H * 4,
                                              (size_t)H * 4, (size_t)R, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
          return DFLASH_ERR_CUDA;
    }
    // final norm (deferred) -> LM head, every row's logits stored
    GemmSpec lm = spec_lm(ctx, R);
    lm.epi.kind = EPI_STORE;
    lm.epi.out[0] = d_logits;
    lm.epi.ld_out[0] = c.vocab;
    lm.epi.rows_per_req = n;
    if (c.n_layers == 0)
      DFL_CHECK(cuda_status(launch_rmsnorm(ctx->x, R, H, ctx->final_norm, c.rms_eps, ctx->h, 0, nullptr, st,
                                           ctx->use_pdl),
                            "rmsnorm launch"));
    return run_gemm(ctx, lm, st);
  } catch (...) {   // no C++ exception crosses the C ABI
    return DFLASH_ERR_OOM;
  }
}

extern "C" dflash_status dflash_spec_commit(int bs, int B, const int* d_draft, const int* d_accepted,
                                            const int* d_next_token, int* d_out_tokens, int max_out, int* d_out_len,
                                            int* d_anchor, int* d_ctx_len, int* d_n_new, int* d_start_pos,
                                            void* stream) {
  if (bs <= 0 || B <= 0 || max_out <= 0 || (B > 1 && !d_draft) || !d_accepted || !d_next_token || !d_out_tokens ||
      !d_out_len || !d_anchor || !d_ctx_len || !d_n_new || !d_start_pos)
    return DFLASH_ERR_ARG;
  return cuda_status(launch_spec_commit(bs, B, d_draft, d_accepted, d_next_token, d_out_tokens, max_out, d_out_len,
                                        d_anchor, d_ctx_len, d_n_new, d_start_pos,
                                        reinterpret_cast<cudaStream_t>(stream)),
                     "spec commit launch");
}
