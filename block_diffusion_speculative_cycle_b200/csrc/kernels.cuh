// Launch interfaces of the non-GEMM kernels of the draft cycle.
#pragma once

#include "common.cuh"

namespace dfl {

struct AttnParams {
  const void* q;              // [R, n_q*d] block queries (RoPE applied)
  const void* kblk;           // [R, n_kv*d] block keys (RoPE applied)
  const void* vblk;           // [R, n_kv*d] block values
  const void* kc;             // cache pool [num_pages, n_kv, page_size, d]
  const void* vc;
  const int* ctx_len;         // [bs]
  const int* page_table;      // [bs, max_pages]
  int max_pages, num_pages, page_size;
  int bs, B, n_q, n_kv, d, g;
  int kps;                    // keys per split (the last split also takes the keys past n_splits*kps)
  int n_splits;
  int ks;                     // tensor-core path: key groups per CTA (1, or 2 for <= 64 query rows)
  int max_ctx;
  float scale;                // 1/sqrt(d)
  float* part_o;              // [bs, n_kv, n_splits, g*B, d]
  float* part_m;              // [bs, n_kv, n_splits, g*B]
  float* part_l;
  int* status;
  size_t out_plane;           // tensor-core path: elements from the output's hi plane to its lo plane
  int cache_f16;              // tensor-core path: the cache pools hold fp16 (else bf16, converted on load)
  int global_merge;           // tensor-core path: splits write part_o/m/l (exp2 domain) and a second kernel merges
  int window;                 // sliding window: the block sees context positions P-window .. P-1 only (0: all)
  int causal;                 // fp32 path only: block row i sees block keys 0..i (a causal decoder), not all B
  // Global merge with a split size chosen on the device (tensor-core path; null:
  // kps above): [keys per split, the batch's (request, split) items], written by
  // the call's embedding kernel from every request's context length (AttnKpsPlan).
  const int* kps_dev;
};

// The device-side split size of a batch, from every request's key tiles t_r (its
// window's 64-aligned start to P, plus the B block keys): among candidate sizes c
// (the longest request cut into 1..16 parts, and the batch's tiles spread over
// 1..4 waves of CTA slots), the one with the fewest waves x (start-up + c tiles),
// waves = ceil(n_kv * sum_r ceil(t_r / c) / slots); never below min_tiles, which
// bounds the grid. Ragged batches get short, equal CTAs; uniform ones one wave.
struct AttnKpsPlan {
  const int* ctx_len;   // [bs]
  int bs, B, window, max_ctx;
  int min_tiles;        // smallest split (key tiles) the grid and workspace allow
  int slots, n_kv;      // CTAs resident at once; KV heads (CTAs per item)
  int* out;             // [2]: keys per split, the batch's (request, split) items; null: no plan
};
constexpr int kAttnPlanStartTiles = 4;   // a CTA's start-up (Q, first tiles, merge) in key tiles

// Keys per split of the call (kps_dev set), else the host's.
__device__ __forceinline__ int attn_kps(const AttnParams& p) { return p.kps_dev ? __ldg(p.kps_dev) : p.kps; }

// First context key the block attends to, and the 64-aligned key where split 0
// starts (keys from there up to ctx_lo are masked; a 64-key tile never crosses a
// page of a multiple of 64 keys, so the tile stays inside ctx_lo's page).
__device__ __forceinline__ int attn_ctx_lo(int P, int window) { return window > 0 ? max(0, P - window) : 0; }
__device__ __forceinline__ int attn_key_base(int ctx_lo) { return ctx_lo & ~63; }

// Tensor-core attention for the bf16 drafter (q / block k / block v fp16, cache bf16 or fp16):
// the n_splits CTAs of one (request, KV head) form a cluster and merge through
// distributed shared memory into out [R, n_q*d], written as bf16 hi/lo planes
// out_plane elements apart.
// kps must be a multiple of 64 and n_splits <= kMaxAttnCluster.
constexpr int kMaxAttnCluster = 16;
cudaError_t launch_attn_cluster(const AttnParams& p, void* out, cudaStream_t st, bool pdl);

// Merge of split partials written to global memory (part_o / part_m / part_l,
// exp2 domain) into out [R, n_q*d] as bf16 hi/lo planes (the cluster kernels'
// global-merge mode).
cudaError_t launch_attn_gmerge(const AttnParams& p, void* out, cudaStream_t st, bool pdl);

// Tensor-core (tcgen05) attention for the bf16 drafter with an fp16 cache whose
// page size is a multiple of 64. Tensor maps (fp16, 128-byte swizzle, boxes of
// 64 elements inner):
//   qmap   q [R, n_q, d] as 3D (d, n_q, R), box (64, g, B)
//   kbmap, vbmap  block k / v [bs, B, n_kv*d] as 3D (n_kv*d, B, bs), box (64, 64, 1)
//   kcmap, vcmap  this layer's cache pools as 2D (d, num_pages*n_kv*page_size), box (64, 64)
constexpr int kMaxAttnTcStages = 6;
struct alignas(64) AttnTcParams {
  CUtensorMap qmap, kbmap, vbmap, kcmap, vcmap;
  AttnParams a;
  int stages;                 // K/V ring depth of the full form (2..kMaxAttnTcStages; 5 fits with d = 128)
  int compact;                // the compact form: <= 64 query rows, two-stage ring, two CTAs per SM
};
// With a.global_merge set, the caller follows it with launch_attn_gmerge.
cudaError_t launch_attn_tc(const AttnTcParams& tp, void* out, cudaStream_t st, bool pdl);
size_t attn_tc_smem_bytes(int d, bool compact, int stages, int splits, bool gmerge, int nr);
// Clusters of n CTAs (n = 1: single CTAs) of the tensor-core attention kernel that can be resident at once.
int attn_tc_max_clusters(int d, bool compact, int stages, int n, bool gmerge, int nr);

// CUDA-core split-KV attention partials (fp32 path), then the log-sum-exp merge into out [R, n_q*d].
cudaError_t launch_attention(const AttnParams& p, void* out, int out_bf16, int in_bf16, cudaStream_t st, bool pdl);

// x[m] = E[token(m)], h[m] = RMSNorm(x[m]) * gain. token(m) for row m (request m / B,
// position i = m % B): tokens[m] when tokens is given; else the anchor at i = 0 and
// draft[request, i-1] (when draft is given) or the mask id at i >= 1.
// With h_plane != 0 (bf16 h), h is written as hi/lo planes h_plane elements apart.
// Each row's block also fills that row's entries of the RoPE table rf (if rf.out);
// block 0 also computes the call's attention split size (kp.out, if set).
cudaError_t launch_embed_norm(const void* embed, int embed_bf16, const int* anchor, int mask_id, const int* tokens,
                              const int* draft, int B, int R, int V, int H, const float* gain, float eps, float* x, void* h, int h_bf16, size_t h_plane,
                              int* status, const RopeFill& rf, const AttnKpsPlan& kp, cudaStream_t st, bool pdl);
// h[m] = RMSNorm(x[m]) * gain into h (model dtype) and/or y (fp32); either may be null.
cudaError_t launch_rmsnorm(const float* x, int R, int H, const float* gain, float eps, void* h, int h_bf16, float* y,
                           cudaStream_t st, bool pdl);
// Copy the block's k / v rows (fp32 [R, n_kv*d], row m = request m / n, position
// pos0[request] + m % n) into the page pools [num_pages, n_kv, page_size, d];
// rows whose page slot or page id is out of range are skipped and flagged.
cudaError_t launch_kv_scatter(const float* kb, const float* vb, const int* pos0, int n, int R, int n_kv, int d,
                              const int* page_table, int max_pages, int num_pages, int page_size, float* kc, float* vc,
                              int* status, cudaStream_t st);
// Device-side commit of one speculative cycle per request (see dflash_spec_commit).
cudaError_t launch_spec_commit(int bs, int B, const int* draft, const int* accepted, const int* next_token,
                               int* out_tokens, int max_out, int* out_len, int* anchor, int* ctx_len, int* n_new,
                               int* start_pos, cudaStream_t st);
// draft[b, i-1] = index(keys[b*B + i]) for i >= 1; every key reset to 0.
cudaError_t launch_argmax_finalize(unsigned long long* keys, int bs, int B, int* draft, cudaStream_t st, bool pdl);

}  // namespace dfl
