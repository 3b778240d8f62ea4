/*
 * dflash.h — C ABI of the B200 (sm_100a) DFlash draft-cycle library.
 *
 * One draft cycle of block-diffusion speculative decoding has three calls:
 *
 *   dflash_inject_ctx   target features -> per-layer injected K/V in the drafter cache
 *   dflash_draft_block  anchor + cache -> B-1 draft tokens in one non-causal pass
 *   dflash_verify       target block logits + drafts -> accepted length, next token
 *
 * Sources (page title, section):
 *   [P1] "DFlash — 블록 확산 드래프터로 6배 빨라지는 투기적 디코딩": §1 greedy verify,
 *        §2 the cycle (anchor, B-1 masks, one drafter pass, one verify pass) and
 *        KV injection, §6 non-causal in-block attention.
 *   [P2] "한 번에 초안을 생성하는 DFlash ...": features of uniformly spaced target
 *        layers, fused by a lightweight projection, injected into every drafter
 *        layer's Key/Value.
 *   [P3] "기술 요약: DFlash – 플래시 추측적 디코딩을 위한 블록 확산": §2.2 context feature
 *        extraction, KV injection into the drafter's KV cache, parallel block
 *        prediction in one forward pass; §2.3 embedding and LM head shared with
 *        the target and frozen.
 *   [P4] "DFlash 소개" (forum post): the spec_generate(target, draft, input_ids,
 *        num_speculative_tokens, temperature, max_new_tokens) call shape.
 *
 * Conventions for every entry point
 *   - All tensors are caller-owned device memory, row-major, densely packed
 *     unless a leading dimension is given. The library never frees them.
 *   - "stream" is a cudaStream_t (NULL = legacy default stream). Every call is
 *     asynchronous on it and enqueues kernels only: no host synchronisation, no
 *     allocation, so a whole cycle can be captured in a CUDA graph.
 *   - Argument errors are detected on the host before any launch and returned
 *     as DFLASH_ERR_ARG / DFLASH_ERR_UNSUPPORTED; nothing is enqueued then.
 *   - Errors found by kernels (a token id, page id or position out of range; a
 *     bounded device wait that gave up) are recorded in a device status word;
 *     the offending element is skipped, the kernel returns normally, and
 *     dflash_get_error() reports and clears it. Kernels never trap.
 *   - Inputs that change from cycle to cycle (anchor, context length, n_new,
 *     start position) are device pointers, so the host never needs to read
 *     the previous cycle's result.
 *   - Weights and features are bf16 or fp32 (dflash_config.dtype); the KV
 *     cache is the same type or, for a bf16 drafter, fp16
 *     (dflash_config.cache_dtype); RMSNorm gains are always fp32.
 *     Accumulation is fp32; the draft argmax is taken on fp32 logits, which
 *     are never written to memory.
 *   - No C++ exception crosses this interface: a failed host allocation is
 *     returned as DFLASH_ERR_OOM.
 */
#ifndef DFLASH_H
#define DFLASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DFLASH_OK = 0,
  DFLASH_ERR_ARG = 1,          /* invalid argument (host-side check) */
  DFLASH_ERR_CUDA = 2,         /* a CUDA runtime / driver call failed */
  DFLASH_ERR_OOM = 3,          /* device workspace (dflash_create) or host allocation failed */
  DFLASH_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up */
  DFLASH_ERR_DEVICE = 5,       /* a kernel met an out-of-range id, page or position */
  DFLASH_ERR_UNSUPPORTED = 6   /* a shape the library has no kernel for */
} dflash_status;

typedef enum { DFLASH_F32 = 0, DFLASH_BF16 = 1, DFLASH_F16 = 2 } dflash_dtype;

/* Drafter shape. Notation of the pages: B = block size (anchor + B-1 masks). */
typedef struct {
  int hidden;          /* H */
  int n_layers;        /* L (5 for the 8B-class drafters, 8 for the coder drafter) */
  int n_q_heads;       /* n_q */
  int n_kv_heads;      /* n_kv; n_q % n_kv == 0, query head j reads kv head j / (n_q/n_kv) */
  int head_dim;        /* d: 64 or 128 */
  int intermediate;    /* SwiGLU width I */
  int vocab;           /* V (shared with the target) */
  int n_feat_layers;   /* n_f: number of tapped target layers */
  int target_hidden;   /* H_t: feature width per tapped layer */
  int mask_token_id;   /* id fed at the B-1 masked positions, 0 <= id < V */
  int max_block;       /* largest B passed to dflash_draft_block / dflash_verify */
  int max_batch;       /* largest bs */
  int max_inject_rows; /* largest bs * max_new passed to dflash_inject_ctx */
  int page_size;       /* tokens per KV page (64 in the batched workloads) */
  float rope_theta;    /* rotary base theta; pair (i, i+d/2) turns by pos * theta^(-2i/d) */
  float rms_eps;       /* RMSNorm epsilon */
  dflash_dtype dtype;  /* storage type of weights and features; DFLASH_F32 or DFLASH_BF16 */
  /* Element type of the drafter's KV cache pools. DFLASH_F16 is accepted for a
   * bf16 drafter: the injected K/V keep 3 more mantissa bits and the attention
   * kernel reads them without conversion (|K|, |V| must stay below 65504). Any
   * other value means "same as dtype" (so a zero-initialised field keeps the
   * model dtype). DFLASH_F16 with an fp32 drafter is rejected (DFLASH_ERR_ARG). */
  dflash_dtype cache_dtype;
  /* Sliding window of the drafter's attention over its cache ("DFlash 소개": the
   * MLX backend bounds the drafter KV cache by a sliding window for long inputs):
   * with window W > 0 the block of a request with context length P attends to
   * context positions max(0, P - W) .. P-1 only (and to the whole block), and
   * never reads the cache below them, so pages that hold only older positions
   * may be released and their page-table slots left as -1. 0: no window. */
  int window;
} dflash_config;

/* Weights: device pointers, [out_features, in_features] row-major, in
 * config.dtype (norm gains: fp32 [H]). Per-layer entries are HOST arrays of
 * n_layers device pointers; the library copies the pointer values at create
 * time and keeps them (the tensors must outlive the context).
 *   fc      [H, n_f*H_t]   lightweight projection of the concatenated features
 *   embed   [V, H]         target-owned token embedding (shared, frozen)
 *   lm_head [V, H]         target-owned LM head (may equal embed)
 *   wq [n_q*d, H], wk/wv [n_kv*d, H], wo [H, n_q*d],
 *   wgate/wup [I, H], wdown [H, I]                                          */
typedef struct {
  const void* fc;
  const void* embed;
  const void* lm_head;
  const float* final_norm;
  const float* const* attn_norm;
  const void* const* wq;
  const void* const* wk;
  const void* const* wv;
  const void* const* wo;
  const float* const* mlp_norm;
  const void* const* wgate;
  const void* const* wup;
  const void* const* wdown;
} dflash_weights;

typedef struct dflash_ctx dflash_ctx;

/* Create a drafter context. Validates the shape, encodes the weights' TMA
 * descriptors and allocates the library's own workspace (activations, split-K
 * partials, argmax keys, a device status word) on the current device.
 * Returns DFLASH_ERR_UNSUPPORTED for shapes without a kernel (bf16 needs H,
 * n_q*d, n_kv*d, I, V multiples of 128 and n_f*H_t a multiple of 64).
 * On success *out owns the context; release it with dflash_destroy. */
dflash_status dflash_create(const dflash_config* cfg, const dflash_weights* w, dflash_ctx** out);

/* Free the context and its workspace (synchronises the device first). NULL is a no-op. */
void dflash_destroy(dflash_ctx* ctx);

/* KV injection ([P3] §2.2, [P2], [P1] §2): c = F · W_fcᵀ, then for every layer l
 * K_l = RoPE(c · Wk_lᵀ) at the row's absolute position and V_l = c · Wv_lᵀ,
 * written into that layer's cache pages. No norm precedes Wk/Wv here.
 *
 *   feats       [bs, max_new, n_f*H_t] (dtype): features of the tapped target
 *               layers, concatenated shallow -> deep; rows >= n_new[r] are ignored
 *   d_n_new     [bs] int32 (device): rows to inject per request, 0..max_new
 *   d_start_pos [bs] int32 (device): absolute position of request r's first row
 *   k_cache, v_cache: HOST arrays [n_layers] of device pointers to page pools
 *               [num_pages, n_kv, page_size, d] (cache_dtype)
 *   d_page_table [bs, max_pages] int32 (device): page of token block p of request r
 * A position whose page slot is beyond max_pages, or whose page id is outside
 * [0, num_pages), is skipped and flagged (DFLASH_ERR_DEVICE). */
dflash_status dflash_inject_ctx(dflash_ctx* ctx, const void* feats, int bs, int max_new,
                                const int* d_n_new, const int* d_start_pos,
                                void* const* k_cache, void* const* v_cache,
                                const int* d_page_table, int max_pages, int num_pages,
                                void* stream);

/* One drafter pass over the block ([P1] §2 steps 1-3, §6; [P3] §2.2):
 * rows (r, i), i < B, hold E[anchor_r] (i = 0) or E[mask_token_id] at position
 * ctx_len[r] + i. Every layer: RMSNorm -> q,k,v (RoPE on q,k) -> attention of
 * each block query over the request's injected context K/V (positions
 * 0..ctx_len[r]-1) and all B block keys, no mask -> Wo + residual; RMSNorm ->
 * SwiGLU MLP + residual. Then the final RMSNorm, the shared LM head and a
 * greedy argmax (lowest id on ties) per masked row, fused: logits are never
 * stored. The block's own K/V are not written to the cache.
 *
 *   d_anchor  [bs] int32 (device): last accepted token per request
 *   d_ctx_len [bs] int32 (device): injected context length P_r, 0 <= P_r <= max_ctx
 *   max_ctx   host upper bound on every P_r (sizes the attention split grid)
 *   d_draft   [bs, B-1] int32 (device, out): d_1..d_{B-1}
 *   d_hidden_out: NULL, or [L+1, bs, B, H] fp32 (device, out): the residual
 *               stream after each layer, then the final normed rows (for parity
 *               checks; costs extra writes). */
dflash_status dflash_draft_block(dflash_ctx* ctx, const int* d_anchor, const int* d_ctx_len, int bs, int B,
                                 const void* const* k_cache, const void* const* v_cache,
                                 const int* d_page_table, int max_pages, int num_pages, int max_ctx,
                                 int* d_draft, float* d_hidden_out, void* stream);

/* Sampled drafting (temperature T > 0; [P1] §1 speculative sampling, [P2] results
 * at temperature 1): the same drafter pass as dflash_draft_block, but each draft
 * token is drawn from softmax(logits_i / T) by the Gumbel-max rule,
 *   d_i = argmax_v (logits_i[v] / T - log(-log u_i[v])),
 * fused into the LM head, and the drafter's logits are stored for the sampled
 * verify (its q). The uniforms are Philox4x32-10 (Salmon et al., SC 2011) under
 * key `seed`: for request r, position i (1..B-1) and vocabulary entry v, word
 * (v mod 128) div 32 of the block at counter (v div 128, v mod 32, i, r), mapped
 * to ((word >> 9) + 1/2) / 2^23. Pass a new seed per cycle for independent draws.
 *   temperature    > 0 and finite (DFLASH_ERR_ARG otherwise)
 *   d_draft_logits [bs, B-1, V] fp32 (device, out): logits of positions 1..B-1
 * Other arguments, outputs and errors as for dflash_draft_block. */
dflash_status dflash_draft_block_sample(dflash_ctx* ctx, const int* d_anchor, const int* d_ctx_len, int bs, int B,
                                        const void* const* k_cache, const void* const* v_cache,
                                        const int* d_page_table, int max_pages, int num_pages, int max_ctx,
                                        float temperature, unsigned long long seed, int* d_draft,
                                        float* d_draft_logits, float* d_hidden_out, void* stream);

/* Bytes of scratch dflash_verify needs for (bs, B). */
size_t dflash_verify_workspace_size(int bs, int B);

/* Greedy verify ([P1] §1, §2 step 4): g_j = argmax_v logits[r, j, v] (lowest
 * index on ties, NaN below every number, -0 == +0, compared in fp32);
 * a_r = number of leading i >= 1 with draft[r, i-1] == g_{i-1};
 * next_r = g_{a_r} (the correction, or the bonus token when a_r = B-1).
 * The committed tokens are draft[r, 0..a_r-1] followed by next_r.
 *
 *   d_logits    [bs, B, V] in logits_dtype (device)
 *   d_draft     [bs, B-1] int32 (device)
 *   d_accepted, d_next_token [bs] int32 (device, out)
 *   d_workspace at least dflash_verify_workspace_size(bs, B) bytes of device
 *               memory, zero-filled before its first use; every call leaves
 *               it zero-filled again. Calls that share a workspace must not
 *               overlap on the GPU.
 * Independent of any drafter context. Results are bit-exact given the logits. */
dflash_status dflash_verify(const void* d_logits, dflash_dtype logits_dtype, const int* d_draft,
                            int bs, int B, int V, int* d_accepted, int* d_next_token,
                            void* d_workspace, size_t workspace_bytes, void* stream);

/* Bytes of scratch dflash_verify_sampled needs for (bs, B, V). */
size_t dflash_verify_sampled_workspace_size(int bs, int B, int V);

/* Sampled verify (T > 0; [P1] §1: keep drafts the target agrees with, from the
 * first rejection draw from the target, so the output follows target-only
 * sampling; the standard speculative-sampling rule, position by position).
 * With p_j = softmax(logits[r, j] / T) and q_i = softmax(draft_logits[r, i-1] / T):
 *   draft i (1..B-1) is accepted while u_accept[r, i-1] * q_i(d_i) < p_{i-1}(d_i);
 *   a_r = the number accepted; next_r is drawn from max(0, p_a - q_{a+1}),
 *   normalised (p_a itself if that is zero everywhere), or from p_{B-1} when every
 *   draft passed: the smallest v whose running sum in index order exceeds
 *   u_final[r] times the total.
 *   d_logits       [bs, B, V] target logits in logits_dtype (bf16 or fp32)
 *   d_draft_logits [bs, B-1, V] fp32: the drafter's logits (dflash_draft_block_sample)
 *   d_draft        [bs, B-1] int32; an id outside [0, V) is rejected
 *   d_u_accept     [bs, B-1] fp32, d_u_final [bs] fp32: uniforms in [0, 1) (inputs)
 *   d_workspace    at least dflash_verify_sampled_workspace_size(bs, B, V) bytes,
 *                  256-byte aligned, zero-filled before its first use; every call
 *                  leaves the part that must start at zero zeroed again. Calls that
 *                  share a workspace must not overlap on the GPU.
 * Computed in fp32 with every sum in a fixed order: reproducible run to run. */
dflash_status dflash_verify_sampled(const void* d_logits, dflash_dtype logits_dtype, const float* d_draft_logits,
                                    const int* d_draft, int bs, int B, int V, float temperature,
                                    const float* d_u_accept, const float* d_u_final, int* d_accepted,
                                    int* d_next_token, void* d_workspace, size_t workspace_bytes, void* stream);

/* Verify for callers that cannot allocate device memory. Same computation,
 * outputs and bit-exact results as dflash_verify; the pages have no
 * counterpart, this is a deployment convenience. Some callers may not call
 * cudaMalloc at all: an inference server's custom-operator interface that hands
 * a kernel only its input and output buffers, or a serving loop whose memory
 * pool has already claimed the GPU's free memory for the KV cache, where a raw
 * cudaMalloc can fail and also synchronises the device, stalling every stream.
 * This variant keeps its scratch in one fixed array compiled into the library:
 * DFLASH_VERIFY_NOALLOC_MAX_ROWS 64-bit keys plus DFLASH_VERIFY_NOALLOC_MAX_BATCH
 * 32-bit tickets (36 KB), present on every GPU that loads the library and held
 * until the process exits.
 *   - The first call on a device looks up the array's device address with that
 *     device current; make that first call before any stream capture.
 *   - Each call clears the part of the array it uses (cudaMemsetAsync on
 *     `stream`) before its kernel runs.
 *   - All calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race and
 *     give wrong results; serialise them.
 *   - bs > DFLASH_VERIFY_NOALLOC_MAX_BATCH or bs*B > DFLASH_VERIFY_NOALLOC_MAX_ROWS
 *     is rejected with DFLASH_ERR_ARG and a message on stderr; other arguments
 *     as for dflash_verify. It allocates nothing. */
#define DFLASH_VERIFY_NOALLOC_MAX_ROWS 4096
#define DFLASH_VERIFY_NOALLOC_MAX_BATCH 1024
dflash_status dflash_verify_noalloc(const void* d_logits, dflash_dtype logits_dtype, const int* d_draft,
                                    int bs, int B, int V, int* d_accepted, int* d_next_token, void* stream);

/* A causal target forward for the speculative loop on the device ([P4] "DFlash
 * 소개": spec_generate(target, draft, ...); [P1] §1-2: the target verifies the
 * block in one forward pass and its features feed the drafter). The context must
 * come from dflash_create with the TARGET's weights, fp32 (DFLASH_ERR_UNSUPPORTED
 * for bf16); `fc` and the feature fields are not used. It runs the same layer
 * (pre-norm RMSNorm, GQA with RoPE, SwiGLU) causally over n rows per request:
 * row i of request r is position pos0[r] + i and attends to the target cache's
 * positions < pos0[r] and to rows 0..i; its own K/V are written into the cache
 * (so rows past the accepted ones are simply overwritten later: truncation is
 * the caller's context length). No sliding window.
 *   d_tokens   [bs, n] int32, or NULL: row 0 = d_anchor[r], row i = d_draft[r, i-1]
 *              (the verify block [anchor, d_1 .. d_{n-1}])
 *   d_pos0     [bs] int32 (device): position of each request's row 0
 *   k_cache, v_cache, d_page_table, max_pages, num_pages: the target's own page
 *              pools and table (layout as for dflash_inject_ctx)
 *   max_ctx    host bound on every pos0: the attention split plan depends on bs and
 *              max_ctx only, so with the same max_ctx a row's logits are the same
 *              bits in a block forward and in a one-row forward
 *   taps       HOST array of n_taps ascending layer indices; d_feats [bs, n, n_taps*H]
 *              fp32 (out) receives the residual stream after each tapped layer,
 *              concatenated shallow to deep (the drafter's injection features)
 *   d_logits   [bs, n, V] fp32 (out) */
dflash_status dflash_target_forward(dflash_ctx* ctx, const int* d_tokens, const int* d_anchor, const int* d_draft,
                                    int bs, int n, const int* d_pos0, void* const* k_cache, void* const* v_cache,
                                    const int* d_page_table, int max_pages, int num_pages, int max_ctx,
                                    const int* taps, int n_taps, float* d_logits, float* d_feats, void* stream);

/* Device-side control of the speculative loop ([P1] §2 steps 1-4 and §1: the
 * accepted drafts and the correction are committed). Per request r, after
 * dflash_verify gave (a, next) for the block drafted at context length P = ctx_len[r]:
 * appends draft[r, 0..a-1] and next to out_tokens[r, out_len[r] ..] (at most
 * max_out tokens per request), then sets start_pos[r] = P, n_new[r] = a + 1 (the
 * committed block rows whose target features are injected next), ctx_len[r] = P + a + 1
 * and anchor[r] = next. All arrays are device int32 [bs] ([bs, max_out] for
 * out_tokens, [bs, B-1] for draft); nothing is read back to the host. */
dflash_status dflash_spec_commit(int bs, int B, const int* d_draft, const int* d_accepted, const int* d_next_token,
                                 int* d_out_tokens, int max_out, int* d_out_len, int* d_anchor, int* d_ctx_len,
                                 int* d_n_new, int* d_start_pos, void* stream);

/* Dynamic block-size scheduling ([P3] §3 item 4 and §4: the drafter trained
 * with block 16 also runs with smaller blocks, the block size scheduled
 * dynamically). Reading taken: per-position acceptance rates
 * alpha_i = P(draft i accepted | drafts 1..i-1 accepted), estimated from verify
 * results with decayed counts and a Beta(1, 1) prior, alpha_i = (A_i + 1) / (T_i + 2);
 * a cycle with block B commits 1 + sum_{i<B} prod_{j<=i} alpha_j tokens on
 * average; the policy picks the candidate B with the most expected tokens per
 * unit of the caller's cycle cost (the smaller B on an exact tie).
 *
 * dflash_acceptance_count: device side of the estimate. For each request r of a
 * cycle run with block B (d_accepted [bs] int32, device, e.g. dflash_verify's
 * output), adds 1 to d_counts[i] (tested) for positions 1 <= i <= min(a_r+1, B-1)
 * and 1 to d_counts[n_pos + i] (accepted) for 1 <= i <= a_r. d_counts is a device
 * array [2 * n_pos] of uint64 that the caller zero-fills and reads (integer
 * atomics: exact and order-independent). B must not exceed n_pos. */
dflash_status dflash_acceptance_count(const int* d_accepted, int bs, int B, unsigned long long* d_counts,
                                      int n_pos, void* stream);

/* Host-side policy (no GPU work). candidates: block sizes 1..n_pos to choose
 * among; decay in (0, 1]: weight kept by past counts at each observation. */
typedef struct dflash_block_policy dflash_block_policy;
dflash_status dflash_block_policy_create(const int* candidates, int n_candidates, double decay, int n_pos,
                                         dflash_block_policy** out);
void dflash_block_policy_destroy(dflash_block_policy* policy);
/* Fold one window of counts in (host copies of the two halves of d_counts above):
 * T_i <- decay * T_i + tested[i], A_i <- decay * A_i + accepted[i]. */
dflash_status dflash_block_policy_observe(dflash_block_policy* policy, const unsigned long long* tested,
                                          const unsigned long long* accepted, int n_pos);
/* Expected tokens committed by a cycle with block B (-1 for a B outside 1..n_pos). */
double dflash_block_policy_expected_tokens(const dflash_block_policy* policy, int B);
/* The candidate maximising expected tokens / costs[k] (costs in the candidates'
 * ascending order, each > 0; e.g. measured cycle times at the current
 * concurrency); a negative dflash_status on bad arguments. */
int dflash_block_policy_choose(const dflash_block_policy* policy, const double* costs, int n_costs);
/* The same with the cost model c0 + c1 * bs * B (c0: the cycle's fixed cost, c1:
 * the cost of verifying one more token of one request). */
int dflash_block_policy_choose_linear(const dflash_block_policy* policy, int bs, double c0, double c1);

/* Per-kernel timing, an instrumentation hook with no counterpart on the pages.
 * While enabled, every kernel this context launches is bracketed by a pair of
 * CUDA events on its stream, tagged with the launch's algorithmic bytes (each
 * weight, activation and output element counted once) and flops. Meant for
 * eager (not graph-captured) profiling passes: it adds event records between
 * launches. dflash_profile_read synchronises, aggregates per kernel kind and
 * clears the records. */
typedef struct {
  char name[32];      /* kernel kind: "gemm_tc", "gemm_simt", "attention", "rmsnorm", ... */
  int launches;
  double total_ms;    /* summed event-to-event durations */
  double bytes;       /* algorithmic bytes summed over the launches */
  double flops;       /* algorithmic flops summed over the launches */
} dflash_profile_entry;

dflash_status dflash_profile_enable(dflash_ctx* ctx, int enable);

/* Fill up to max_entries aggregated entries; returns how many were written
 * (negative dflash_status on error). Resets the records. */
int dflash_profile_read(dflash_ctx* ctx, dflash_profile_entry* out, int max_entries);

/* GEMM-chain instrumentation, no counterpart on the pages. Enqueues on `stream`,
 * back to back, exactly the tensor-core GEMM launches one cycle of this shape
 * makes, with the same plans, fused epilogues and programmatic dependent
 * launch, and nothing else: the injection's two (as dflash_inject_ctx, with the
 * same arguments and effect on the cache), then per layer QKV, O, gate/up and
 * down, then the LM head (R = bs * B rows, positions from d_ctx_len). Its purpose
 * is timing the GEMMs as they run inside a cycle, overlapping each other's ramp
 * and tail, e.g. by capturing the call in a CUDA graph and timing its replays.
 * The draft-side results are not a draft: the context's activations and residual
 * stream are left unspecified (the next dflash_draft_block rebuilds them) and the
 * argmax state is cleared at the end. bf16 drafters only (DFLASH_ERR_UNSUPPORTED
 * otherwise); argument errors as for dflash_inject_ctx / dflash_draft_block. */
dflash_status dflash_profile_gemm_chain(dflash_ctx* ctx, const void* feats, int bs, int max_new,
                                        const int* d_n_new, const int* d_start_pos, void* const* k_cache,
                                        void* const* v_cache, const int* d_page_table, int max_pages, int num_pages,
                                        const int* d_ctx_len, int B, void* stream);

/* Synchronise `stream`, read and clear the context's device status word.
 * Returns DFLASH_ERR_TIMEOUT, DFLASH_ERR_DEVICE or DFLASH_OK. */
dflash_status dflash_get_error(dflash_ctx* ctx, void* stream);

/* Static, human-readable name of a status code. */
const char* dflash_status_string(dflash_status s);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_H */
