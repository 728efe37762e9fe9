/*
 * vs.h - C ABI of the B200 (sm_100a) sparse-prefill library.
 *
 * One attention layer of a GQA model, prefilled in chunks over a growing KV
 * cache, with vertical-slash sparse attention, attention-recall refinement and
 * Dual Chunk Attention (DCA) position remapping, as described in the Qwen2.5-1M
 * report explainer (0h-n0.github.io/posts/paper-2501-15383): sections "Length
 * Extrapolation" (DCA), "Sparse Attention" (vertical-slash steps), "Chunked
 * Prefill", "Sparsity Refinement" (attention recall) and "Algorithm:
 * integrating DCA and sparse attention" (the chunk loop of
 * sparse_attention_with_dca(query, key, value, chunk_size, last_q)). RoPE
 * follows the rotary code of the long-context essay (deepseekmodel.com,
 * section 2.4): inverse frequencies 1/base^(2m/d), rotate-half pairs (m, m+d/2).
 *
 * Conventions shared by every call:
 *  - Tensors are bf16 (passed as uint16_t bit patterns), head-major and
 *    contiguous: [heads][rows][128]. head_dim must be 128. Base addresses must
 *    be 16-byte aligned. "rows" arguments give the per-head row count (the head
 *    stride in rows). Q and K are passed PRE-RoPE; the library rotates them.
 *  - All pointers are device pointers unless marked (host).
 *  - Every call is asynchronous on the given stream. Argument errors are
 *    detected on the host, return a status and enqueue nothing.
 *  - Ownership: the caller allocates the workspace and every input and output.
 *    The library allocates no device memory (context creation allocates only a
 *    small host struct).
 *  - Device-side failures (a bounded wait that ran out, an index check) set an
 *    error word in the workspace; vs_status_poll() returns and clears it.
 *  - The context keeps rotated copies of K (continuous positions, and DCA key
 *    positions when enabled) in its workspace and extends them as e grows. Rows
 *    [0, e) of k must not change between calls that pass the same k pointer
 *    (an append-only KV cache); call vs_context_reset() before reusing the
 *    buffer for other contents. Every call that reuses a cached rotation
 *    re-rotates 8 rows spread over it and compares them with the cache; a
 *    difference is reported by vs_status_poll() as VS_ERR_DEVICE_CHECK.
 *  - Not thread-safe per context; distinct contexts are independent.
 */
#ifndef VS_H_
#define VS_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define VS_API __attribute__((visibility("default")))
#else
#define VS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VS_OK = 0,
  VS_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or range */
  VS_ERR_UNSUPPORTED = 2,  /* head_dim != 128, Hq % Hkv != 0, sizes beyond the context */
  VS_ERR_WORKSPACE = 3,    /* workspace missing or smaller than vs_workspace_size() */
  VS_ERR_CUDA = 4,         /* a CUDA runtime call failed (message in vs_last_error) */
  VS_ERR_TIMEOUT = 5,      /* a bounded device wait ran out (from vs_status_poll) */
  VS_ERR_DEVICE_CHECK = 6  /* a device-side check failed, e.g. an output list cap */
} vs_status;

typedef struct {
  int32_t hq;              /* query heads */
  int32_t hkv;             /* KV heads; hq % hkv == 0, query head h reads KV head h / (hq/hkv) */
  int32_t head_dim;        /* must be 128 */
  int32_t last_q;          /* estimation rows per chunk, 1..64 (the pages use 64) */
  float softmax_scale;     /* multiplies q.k; 1/sqrt(128) (a YaRN temperature 1/t folds in here) */
  double rope_base;        /* RoPE base (1e7 for the Qwen2.5-1M models) */
  int32_t dca_enabled;     /* 0: continuous positions in attention; 1: DCA positions */
  int64_t dca_chunk_size;  /* DCA chunk size C (the largest relative position is C-1) */
  int64_t dca_local_window;/* DCA local window W, 0 <= W < C; chunk stride S = C - W */
  int32_t refine_dca_positions; /* 0: vs_refine measures recall with continuous positions
                           (the pages' selection positions); 1 (DCA enabled only): recall from
                           the estimation rows' attention at DCA positions, the attention the
                           prefill computes. Needs S % 128 == 0 and the estimation rows inside
                           one DCA chunk, else vs_refine returns VS_ERR_UNSUPPORTED. */
} vs_attn_cfg;

typedef struct vs_ctx vs_ctx;

/* Device workspace needed for sequences of up to max_seq keys and prefill
 * calls of up to max_chunk query rows. */
VS_API vs_status vs_workspace_size(const vs_attn_cfg* cfg, int64_t max_seq, int64_t max_chunk,
                            size_t* bytes /* host */);

/* Creates a context over a caller-owned device workspace (>= vs_workspace_size
 * bytes, 256-byte aligned). Initialises the workspace on `stream`. */
VS_API vs_status vs_context_create(const vs_attn_cfg* cfg, int64_t max_seq, int64_t max_chunk,
                            void* workspace, size_t ws_bytes, cudaStream_t stream,
                            vs_ctx** out /* host */);
VS_API vs_status vs_context_destroy(vs_ctx* ctx);
/* Forgets the cached rotated keys (call when the KV buffer's rows change). */
VS_API vs_status vs_context_reset(vs_ctx* ctx);
/* Wall-time limit (ns) of every bounded device wait; default 2e9. */
VS_API vs_status vs_set_wait_limit(vs_ctx* ctx, uint64_t ns);
/* Summation order of vs_sparse_prefill (default off). Off: a CTA whose work list has
 * 1024 entries or more starts its sweep where the CTAs of its KV head are loading now
 * and wraps around, so that the CTAs in flight share each K/V block in L2 once a
 * KV head's keys and values outgrow it; the online softmax then adds the blocks in an
 * order that depends on timing, and results may differ in the last bits from run to
 * run (each within the same rounding bounds). On: every list is swept from its start
 * and results are bitwise reproducible. VS_ERR_INVALID_ARG for a NULL context. */
VS_API vs_status vs_set_deterministic(vs_ctx* ctx, int on);

/*
 * dca_remap - the DCA position tables for positions t = pos0 .. pos0+n-1
 * ("Length Extrapolation": intra-chunk, inter-chunk and successive-chunk
 * attention). With stride S = C - W and r(t) = t mod S:
 *   pk[t]       = r(t)                 key position
 *   pq_intra[t] = r(t)                 query position against keys of its own chunk
 *   pq_succ[t]  = min(r(t) + S, C - 1) against keys of the previous chunk
 *   pq_inter[t] = C - 1                against keys two or more chunks back
 * With DCA disabled every table holds t itself. Outputs are int32 [n].
 */
VS_API vs_status dca_remap(vs_ctx* ctx, int64_t pos0, int64_t n, int32_t* pk, int32_t* pq_intra,
                    int32_t* pq_succ, int32_t* pq_inter, cudaStream_t stream);

/*
 * vs_estimate - vertical and slash importance of one chunk ("Sparse Attention"
 * step 2, "Chunked Prefill": the last queries of each chunk; "Algorithm": with
 * continuous positions). For the estimation rows R = [max(q_pos0, e-last_q), e)
 * and keys j < e, with A the causal row softmax of softmax_scale * RoPE(q_i, i) .
 * RoPE(k_j, j):
 *   lse[h][r]    = log sum_{j<=i} exp(s_ij) for the r-th row of R   ([hq][64] fp32)
 *   vert[h][j]   = sum_{i in R} A_ij, j in [0, e)                   ([hq][e_ld] fp32)
 *   slash[h][d]  = sum_{i in R, i>=d} A_{i,i-d}, d in [0, e)        ([hq][e_ld] fp32)
 * q: [hq][q_rows][128], row r holding position q_pos0 + r; R must lie in it.
 * k: [hkv][k_rows][128], row j holding position j; e <= k_rows, e <= max_seq.
 */
VS_API vs_status vs_estimate(vs_ctx* ctx, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                      const uint16_t* k, int64_t k_rows, int64_t e, float* vert, float* slash,
                      int64_t e_ld, float* lse, cudaStream_t stream);

/*
 * vs_select - critical tokens of the vertical-slash pattern ("Sparse Attention"
 * step 3): per head the kv_budget[h] columns j with the largest vert and the
 * ks_budget[h] offsets d with the largest slash, offset 0 always included;
 * budgets are capped at e. Ranking: score descending, then index ascending.
 * Outputs ascending: v_idx [hq][cap_v], v_cnt [hq], s_off [hq][cap_s], s_cnt [hq].
 * A list longer than its cap is truncated and raises VS_ERR_DEVICE_CHECK in
 * vs_status_poll. Budgets are device int32 [hq].
 */
VS_API vs_status vs_select(vs_ctx* ctx, const float* vert, const float* slash, int64_t e_ld, int64_t e,
                    const int32_t* kv_budget, const int32_t* ks_budget, int32_t* v_idx,
                    int32_t cap_v, int32_t* v_cnt, int32_t* s_off, int32_t cap_s, int32_t* s_cnt,
                    cudaStream_t stream);

/*
 * vs_refine - sparsity refinement by attention recall ("Sparsity Refinement"):
 * recall_h = mean over the estimation rows of exp(lse_sparse - lse_full), i.e.
 * the softmax mass (continuous positions) that the selected keys cover. While
 * recall_h < tau and a budget is below e, both budgets double (capped at e),
 * at most max_iters times. kv_budget/ks_budget hold the base budgets on entry
 * and the final ones on exit; recall [hq] fp32 gets the final recall; the final
 * sets are written as in vs_select. q, k, vert, slash and lse are those of the
 * preceding vs_estimate call for the same chunk.
 */
VS_API vs_status vs_refine(vs_ctx* ctx, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                    const uint16_t* k, int64_t k_rows, int64_t e, const float* vert,
                    const float* slash, int64_t e_ld, const float* lse, float tau,
                    int32_t max_iters, int32_t* kv_budget, int32_t* ks_budget, int32_t* v_idx,
                    int32_t cap_v, int32_t* v_cnt, int32_t* s_off, int32_t cap_s, int32_t* s_cnt,
                    float* recall, cudaStream_t stream);

/*
 * vs_calibrate_accumulate - the offline form of sparsity refinement ("Sparsity
 * Refinement": the budgets are improved once, on a calibration sequence): after
 * vs_refine has refined one calibration chunk from the base budgets, each head keeps
 * the larger of its accumulated and its refined budgets,
 *   kv_acc[h] = max(kv_acc[h], kv_budget[h]),  ks_acc[h] = max(ks_acc[h], ks_budget[h]).
 * All four are device int32 [hq]; the caller initialises the accumulators (e.g. to 0)
 * and passes them, once every calibration chunk is in, as the fixed budgets of
 * vs_select for every chunk of later sequences.
 */
VS_API vs_status vs_calibrate_accumulate(vs_ctx* ctx, const int32_t* kv_budget, const int32_t* ks_budget,
                                  int32_t* kv_acc, int32_t* ks_acc, cudaStream_t stream);

/*
 * vs_sparse_prefill - attention of the chunk rows i in [q_pos0, e) over the
 * keys j <= i selected by the vertical-slash sets ("Sparse Attention" step 4;
 * "Algorithm": attention with DCA positions):
 *   O_i = sum_{j in M_i} softmax_j(s_ij) v_j,  M_i = {j <= i : j in V or i-j in S}
 * s_ij = softmax_scale * RoPE(q_i, P_q) . RoPE(k_j, P_k) with P_q = i, P_k = j,
 * or the DCA positions of dca_remap when enabled. Query head h reads KV head
 * h / (hq/hkv). q: [hq][q_rows][128] (row r at position q_pos0 + r, e - q_pos0
 * <= q_rows <= max_chunk); k, v: [hkv][kv_rows][128]; out: [hq][q_rows][128]
 * bf16 (rows of the chunk written, others untouched); lse_out: nullable
 * [hq][q_rows] fp32 natural-log softmax normaliser of each row. The order in
 * which the blocks of a long work list are added follows the other CTAs in
 * flight (see vs_set_deterministic), so results may differ in the last bits
 * from run to run unless the context is set deterministic.
 */
VS_API vs_status vs_sparse_prefill(vs_ctx* ctx, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                            int64_t e, const uint16_t* k, const uint16_t* v, int64_t kv_rows,
                            const int32_t* v_idx, int32_t cap_v, const int32_t* v_cnt,
                            const int32_t* s_off, int32_t cap_s, const int32_t* s_cnt,
                            uint16_t* out, float* lse_out, cudaStream_t stream);

/* Counters of the last vs_sparse_prefill on this context (synchronises the
 * stream): [0] executed 128-query x 128-key tiles summed over heads (a tile is a
 * key block, or a group of up to 128 selected vertical columns gathered from key
 * blocks the call does not execute), [1] selected (useful) query-key pairs summed
 * over heads. */
VS_API vs_status vs_prefill_stats(vs_ctx* ctx, cudaStream_t stream, int64_t* out2 /* host [2] */);

/* Measurement hook: when both events are non-NULL, every following
 * vs_sparse_prefill records `start` right before and `stop` right after its
 * attention kernel, on the call's stream (pass NULL, NULL to stop). */
VS_API vs_status vs_set_prefill_events(vs_ctx* ctx, cudaEvent_t start, cudaEvent_t stop);

/*
 * vs_select_noalloc - the selection of vs_select for callers that cannot
 * allocate device memory. (The paper has no counterpart: this is a deployment
 * variant of vs_select, not a step of the method.)
 *
 * Who needs it: code that may not create a workspace, e.g. a plugin running
 * inside an application that owns all device memory through its own arena, or
 * a service that plans its memory at start-up and allows no later cudaMalloc.
 * It takes no context: hq query heads, vert/slash [hq][e_ld] fp32, budgets and
 * outputs exactly as in vs_select, except that cap_v and cap_s must be >= e.
 * Scratch (thresholds and per-element levels) lives in a static device array
 * of 32 MiB per device, held by every GPU that loads the library until exit;
 * hq * 2 * round_up(e, 128) bytes of levels plus, per head, about 2 KB and 2 KB per
 * selection segment (at most 64 segments; 11 at 28 heads) must fit, else
 * VS_ERR_UNSUPPORTED. Nothing is allocated. The first call on a device looks up
 * the array's device address (make it before any stream capture begins); the
 * lookup is repeated when another CUDA context is current on that device, e.g.
 * after cudaDeviceReset. Calls on one device share the array: calls whose
 * kernels overlap on the GPU race.
 */
VS_API vs_status vs_select_noalloc(int32_t hq, const float* vert, const float* slash,
                                   int64_t e_ld, int64_t e, const int32_t* kv_budget,
                                   const int32_t* ks_budget, int32_t* v_idx, int32_t cap_v,
                                   int32_t* v_cnt, int32_t* s_off, int32_t cap_s, int32_t* s_cnt,
                                   cudaStream_t stream);

/* Number of kernels this library has launched in the process so far. */
VS_API uint64_t vs_kernel_launches(void);

/* Synchronises the stream, returns and clears the device error word
 * (VS_OK, VS_ERR_TIMEOUT or VS_ERR_DEVICE_CHECK). */
VS_API vs_status vs_status_poll(vs_ctx* ctx, cudaStream_t stream);

/* Launches a kernel whose bounded wait is given an mbarrier that nothing
 * completes, with the given limit (ns); the following vs_status_poll must
 * report VS_ERR_TIMEOUT and the context stays usable. Exercises the
 * failure path of every wait without faulting the GPU. */
VS_API vs_status vs_selftest_wait_timeout(vs_ctx* ctx, uint64_t limit_ns, cudaStream_t stream);

/* Message of the last error on this thread (never NULL). */
VS_API const char* vs_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VS_H_ */
