/*
 * sla.h - C ABI of the block-routed sparse+linear attention layer (SLA / SALAD
 * style) for NVIDIA B200 (sm_100a).
 *
 * One layer computes, per (batch b, query head h, query block i of 64 tokens):
 *
 *   1. block pooling      qbar_i = mean of the valid Q tokens of block i,
 *                         kbar_j = mean of the valid K tokens of block j
 *                         (SLA analysis, arXiv 2509.24006: compressed attention
 *                          prediction by mean pooling; 2025 sparse-attention
 *                          review, section 11 SpargeAttn, prediction algorithm)
 *   2. pooled scores      s_ij = qbar_i . kbar_j * scale, P_hat = softmax_j(s_i.)
 *                         (same SpargeAttn passage)
 *   3. routing            SLA_MODE_THREEWAY: the k_h highest-scoring blocks of
 *                         row i are critical, the k_l lowest negligible, the
 *                         rest marginal (SLA analysis: critical / marginal /
 *                         negligible split, TopK / BottomK; 2025 review,
 *                         section 10 SLA).  Equal scores: lower block index
 *                         ranks higher.
 *                         SLA_MODE_TOPN_WINDOW: the query heads of one KV group
 *                         sum their per-head softmax over past blocks j < i and
 *                         keep the top_n, plus a causal window of `window`
 *                         tokens (2025 review, section 4 MoBA; sparse attention
 *                         survey, section 2 NSA: block 64, n = 16, w = 512).
 *   4. sparse attention   O_s = exact softmax attention over the valid tokens of
 *                         the critical blocks (top-n mode: selected blocks
 *                         union window, causal); 0 when the set is empty
 *                         (2025 review, section 2.3 NSA operator design).
 *   5. linear attention   h_j = phi(K_j)^T V_j, z_j = sum_t phi(k_t) over valid
 *                         tokens, phi = elu + 1; S_i = sum over marginal j of
 *                         h_j, Z_i likewise; O_l = phi(q) S_i / (phi(q) . Z_i),
 *                         0 when row i has no marginal block
 *                         (SLA analysis: linear attention at O(N d^2) for the
 *                          marginal part).
 *   6. combine            O = O_s + g * (O_l W_p), g_t = sigmoid(q_t . w_g[h])
 *                         (SLA analysis, Proj paragraph: O = O^s + Proj(O^l);
 *                          SALAD summary: input-dependent gate).
 *                         Without projection W_p = I; without gate g = 1.
 *                         The top-n mode has no linear branch: O = O_s, or
 *                         with nsa_branches the gated sum of NSA's compressed,
 *                         selected and window branches (see nsa_branches).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are dense, row-major, in device memory (the caller allocates and
 *   frees all of them; the library never allocates). The one exception is
 *   sla_forward_host, whose q, k, v and out are in host memory:
 *     q    bf16 [B, H,    N, d]
 *     k, v bf16 [B, H_kv, N, d]
 *     w_p  bf16 [d, d]   (row vector times matrix: O_l W_p), ignored unless has_proj;
 *          [H, d, d] with proj_per_head (head h uses w_p[h])
 *     w_g  bf16 [H, d]   ignored unless has_gate; [H, 3, d] with nsa_branches
 *          (gates of the compressed, selected and window branches)
 *     out  bf16 [B, H, N, d]
 *   Tokens at index >= N_valid are padding: they are left out of pooling,
 *   attention and the linear states, and their output rows are written as 0.
 * - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *   enqueues work on it and returns; nothing synchronises except
 *   sla_check_device_status. sla_forward (and sla_forward_blocks) run the
 *   linear-state stage on a side stream the library creates once per device and
 *   context: forked from `stream` after the pooling pass with an event and joined
 *   back before the aggregation, so the call stays ordered on `stream` as a whole
 *   (also under CUDA-graph capture). The timed and host-buffer entry points run
 *   every stage on their own stream.
 * - `ws` is caller-owned device scratch of at least sla_workspace_bytes(cfg)
 *   bytes, 256-byte aligned. Its contents need no initialisation and are
 *   clobbered. Calls that share one `ws` must not overlap on the GPU.
 * - Errors: invalid arguments (bad config, NULL or misaligned pointers, short
 *   workspace) return SLA_ERR_INVALID_ARG / SLA_ERR_UNSUPPORTED /
 *   SLA_ERR_WORKSPACE before anything is launched. A failed launch returns
 *   SLA_ERR_CUDA. Faults detected on the device (an index out of range, a
 *   bounded wait that ran out) are recorded in a status word inside `ws` and
 *   reported by sla_check_device_status; kernels never trap.
 */
#ifndef SLA_H
#define SLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLA_API __attribute__((visibility("default")))
#else
#define SLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,    /* NULL pointer, inconsistent sizes, misalignment */
  SLA_ERR_UNSUPPORTED = 2,    /* valid but outside what the kernels implement */
  SLA_ERR_WORKSPACE = 3,      /* ws NULL or ws_bytes < sla_workspace_bytes(cfg) */
  SLA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  SLA_ERR_DEVICE_TIMEOUT = 5, /* a device-side bounded wait ran out */
  SLA_ERR_DEVICE_CHECK = 6    /* a device-side range check failed */
} sla_status;

typedef enum {
  SLA_MODE_THREEWAY = 0,      /* critical / marginal / negligible (SLA, SALAD) */
  SLA_MODE_TOPN_WINDOW = 1    /* top_n past blocks per KV group + causal window (NSA / MoBA) */
} sla_mode;

typedef struct {
  int32_t B;        /* batch */
  int32_t H;        /* query heads */
  int32_t H_kv;     /* key/value heads; H % H_kv == 0, head h reads KV head h / (H / H_kv) */
  int32_t N;        /* padded sequence length, a multiple of block */
  int32_t N_valid;  /* valid tokens, N - block < N_valid <= N */
  int32_t d;        /* head dimension: 64 or 128 */
  int32_t block;    /* tokens per block: must be 64 */
  int32_t mode;     /* sla_mode */
  int32_t k_h;      /* THREEWAY: critical blocks per row, 0 <= k_h */
  int32_t k_l;      /* THREEWAY: negligible blocks per row, k_h + k_l <= N / block */
  int32_t top_n;    /* TOPN_WINDOW: selected past blocks per query block, >= 0 */
  int32_t window;   /* TOPN_WINDOW: window tokens t-window+1 .. t, >= 0 */
  int32_t causal;   /* must be 1 in TOPN_WINDOW and 0 in THREEWAY */
  int32_t has_proj; /* THREEWAY: 1 = apply w_p to O_l, 0 = identity */
  int32_t proj_per_head; /* THREEWAY with has_proj: 0 = one w_p [d, d] shared by all heads;
                          * 1 = one per query head, w_p [H, d, d]; needs H_kv == H (the
                          * projection is folded into per-KV-head states), else
                          * SLA_ERR_UNSUPPORTED */
  int32_t has_gate; /* THREEWAY: 1 = g = sigmoid(q . w_g[h]), 0 = g = 1; TOPN_WINDOW: only
                     * with nsa_branches (the branch gates) */
  int32_t smooth_k; /* THREEWAY: 1 = the linear branch uses K minus the mean of the head's
                     * valid key tokens (smooth-K, zero-mean K); routing and the sparse
                     * branch are unchanged by it (each row shifts by a constant) */
  int32_t linear_all; /* THREEWAY: 1 = the linear branch runs over every valid key block
                       * (all tokens) instead of the marginal blocks only */
  int32_t cos_filter; /* 1 = key blocks whose CosSim (mean cosine similarity over all
                       * ordered pairs of their valid tokens) is below cos_theta get a
                       * pooled score of -inf (2025 review, section 11, SpargeAttn):
                       * they rank last and get probability 0 in the top-n softmax */
  float scale;      /* softmax scale of pooled scores and attention; 0 = 1/sqrt(d) */
  float cos_theta;  /* CosSim threshold of cos_filter */
  int32_t nsa_branches; /* TOPN_WINDOW: 1 = NSA's three parallel branches (sparse attention
                         * survey, section 2): compressed, selected and window, each its
                         * own softmax, summed with gates g_b = sigmoid(q . w_g[h][b])
                         * (w_g bf16 [H, 3, d] with has_gate, else g_b = 1); 0 = one
                         * softmax over the selected blocks and the window together */
  int32_t cmp_block;  /* nsa_branches: tokens per compressed block (NSA: 32); compressed
                       * block c is the mean of tokens c*cmp_stride .. + cmp_block - 1
                       * (all valid) and query t attends it when c*cmp_stride + cmp_block
                       * - 1 <= t */
  int32_t cmp_stride; /* nsa_branches: stride between compressed blocks (NSA: 16) */
} sla_config;

/*
 * Checks a configuration without touching any pointer.
 * Sizes: B, H, H_kv, N and d must be >= 1; an empty problem (any of them 0) is
 * SLA_ERR_INVALID_ARG, not a no-op. Limits of the kernels (SLA_ERR_UNSUPPORTED
 * beyond them): N / block <= 4096 key blocks (N <= 262144 tokens, the routing
 * sort's row length) and B * H * N * d <= 2^40 elements; in TOPN_WINDOW mode
 * top_n <= 64 and top_n + (window + 62) / 64 + 1 <= 128 (the flash kernel's
 * block list), and cmp_block, cmp_stride <= 1024 with nsa_branches.
 */
SLA_API sla_status sla_validate_config(const sla_config* cfg);

/* Bytes of device workspace that sla_route / sla_forward need for cfg
 * (0 if cfg is invalid). */
SLA_API size_t sla_workspace_bytes(const sla_config* cfg);

/*
 * Routing only (steps 1-3).
 *   THREEWAY:    mask_out int8  [B, H, nqb, nkb]: 2 critical, 1 marginal, 0 negligible
 *                crit_idx int32 [B, H, nqb, k_h]: critical blocks, ascending
 *                neg_idx  int32 [B, H, nqb, k_l]: negligible blocks, ascending
 *   TOPN_WINDOW: mask_out int8  [B, H_kv, nqb, nkb]: 2 selected, 0 otherwise
 *                crit_idx int32 [B, H_kv, nqb, top_n]: selected blocks ascending,
 *                         padded with -1 when fewer than top_n exist (i < top_n)
 *                neg_idx  unused (may be NULL)
 * mask_out may be NULL; crit_idx may be NULL only when k_h (top_n) is 0 and
 * neg_idx only when k_l is 0. nqb = nkb = N / block.
 */
SLA_API sla_status sla_route(const void* q, const void* k, const sla_config* cfg,
                     int8_t* mask_out, int32_t* crit_idx, int32_t* neg_idx,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * The whole layer (steps 1-6): writes out [B, H, N, d] bf16.
 * w_p may be NULL unless has_proj, w_g may be NULL unless has_gate.
 * mask_out (nullable) receives the routing mask exactly as sla_route writes it.
 */
SLA_API sla_status sla_forward(const void* q, const void* k, const void* v,
                       const void* w_p, const void* w_g, const sla_config* cfg,
                       void* out, int8_t* mask_out,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * sla_forward restricted to the output rows of query blocks [qb_begin, qb_end) of every
 * head of cfg: the block level of db-SP's partitioning (sparse attention survey, db-SP:
 * work split at the head level and the block level so that devices get equal sparse
 * work). A head whose query blocks are split over several calls (or devices) costs each
 * of them its whole routing, key pooling and linear states (the key side of a row needs
 * every key block), while the flash kernel and the aggregation run only for the range.
 *   qb_begin, qb_end   0 <= qb_begin < qb_end <= N / block; qb_begin even, and qb_end even
 *                      or N / block (the flash kernel works on pairs of query blocks);
 *                      else SLA_ERR_INVALID_ARG
 *   out                bf16 [B, H, N, d]: only the rows of the range are written (padding
 *                      rows among them as 0); the others keep their contents
 *   mask_out, ws       as sla_forward (mask_out receives the whole routing mask)
 * The rows written are bit-identical to those of a whole-layer sla_forward. The backward
 * pass reads a whole-layer sla_forward's workspace, not this call's.
 */
SLA_API sla_status sla_forward_blocks(const void* q, const void* k, const void* v,
                                      const void* w_p, const void* w_g, const sla_config* cfg,
                                      int32_t qb_begin, int32_t qb_end, void* out, int8_t* mask_out,
                                      void* ws, size_t ws_bytes, void* stream);

/*
 * sla_forward that also records caller-created CUDA events (cudaEvent_t,
 * passed as void*) on `stream` around its launches: events[0] before the first
 * launch and events[s + 1] after stage s, for s < sla_num_stages(cfg).
 * n_events must be sla_num_stages(cfg) + 1. Used to time each kernel.
 */
SLA_API sla_status sla_forward_timed(const void* q, const void* k, const void* v,
                             const void* w_p, const void* w_g, const sla_config* cfg,
                             void* out, int8_t* mask_out,
                             void* ws, size_t ws_bytes, void* stream,
                             void* const* events, int32_t n_events);

/* Number of stages (one kernel launch each) sla_forward enqueues for cfg, or -1. */
SLA_API int32_t sla_num_stages(const sla_config* cfg);

/* Name of stage s of cfg's pipeline (static string), or NULL. */
SLA_API const char* sla_stage_name(const sla_config* cfg, int32_t s);

/*
 * Synchronises `stream`, reads the device status word in ws and clears it.
 * Returns SLA_OK, SLA_ERR_DEVICE_TIMEOUT, SLA_ERR_DEVICE_CHECK or SLA_ERR_CUDA;
 * *detail (nullable) receives a code naming the kernel and check that failed.
 */
SLA_API sla_status sla_check_device_status(void* ws, void* stream, int32_t* detail);

/*
 * The layer on HOST buffers (the pages have no counterpart: this is the call a
 * user with activations in host memory makes). q_host, k_host and v_host are
 * read from host memory and out_host is written there, in the layouts of
 * sla_forward. Host memory should be page-locked: pageable memory also works,
 * but its copies do not overlap anything.
 *
 * Pipelining: the layer is cut into B * n_chunks units, one batch entry and
 * H_kv / n_chunks KV heads each, with their query heads. Every head's result
 * is independent of the others, so a unit's output is bit-identical to the
 * same rows of one sla_forward call. The inputs of all units are copied in on
 * h2d_stream in order. Each unit runs sla_forward on `stream` as soon as its
 * inputs have arrived, and its output is copied out on d2h_stream as soon as
 * it is done. So the copies of later units overlap the kernels of earlier
 * ones, and the two copy directions overlap each other.
 *
 * w_p and w_g are DEVICE pointers (resident parameters, layouts of
 * sla_forward; NULL unless has_proj / has_gate).
 *
 * dev is a caller-owned device arena of sla_forward_host_device_bytes(cfg,
 * n_chunks) bytes, 256-byte aligned. It holds a status word at offset 0,
 * device copies of q, k, v and out, and one sla_forward workspace per unit.
 * sla_check_device_status(dev, stream, ...) reports the first device-side
 * error of any unit.
 *
 * Ordering: the call's copies start after the work queued on `stream` before
 * the call, and `stream` waits for the last copy out before any later work.
 * So completion of `stream` means out_host is written, and back-to-back calls
 * on the same arena do not race. Distinct non-default streams give the
 * overlap; passing the same stream three times is correct but serial. The
 * call creates and releases its own CUDA events and allocates no memory.
 *
 * Errors: SLA_ERR_INVALID_ARG for a bad configuration, n_chunks < 1 or not
 * dividing H_kv, or a NULL or misaligned (16 bytes) pointer;
 * SLA_ERR_WORKSPACE for a NULL, misaligned or short arena; SLA_ERR_CUDA if
 * a copy, event or launch fails. All checks run before the first copy. After
 * SLA_ERR_CUDA, copies that were already queued may still run: synchronise
 * all three streams before freeing or reusing the host buffers or the arena.
 */
SLA_API size_t sla_forward_host_device_bytes(const sla_config* cfg, int32_t n_chunks);
SLA_API sla_status sla_forward_host(const void* q_host, const void* k_host, const void* v_host,
                                    const void* w_p, const void* w_g, const sla_config* cfg,
                                    void* out_host, int32_t n_chunks, void* dev, size_t dev_bytes,
                                    void* stream, void* h2d_stream, void* d2h_stream);

/*
 * Failure-detection self-test (the pages have no counterpart). Clears the
 * status word at the start of `ws` (any buffer of at least 256 bytes,
 * 256-byte aligned) and launches one small kernel that waits, through the
 * same bounded mbarrier wait every kernel of the library uses, on a barrier
 * that nothing completes. After `limit_ns` (1e3 .. 1e9) the wait gives up, the
 * kernel records SLA_ERR_DEVICE_TIMEOUT with detail 300 in the status word and
 * returns, so sla_check_device_status(ws, ...) then reports the timeout and the
 * GPU context stays usable. Returns SLA_ERR_INVALID_ARG for a bad ws or limit,
 * SLA_ERR_CUDA for a failed launch, else SLA_OK.
 */
SLA_API sla_status sla_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream);

/*
 * Token order along a 3-D Hilbert curve (2025 review, section 11, SpargeAttn:
 * reordering tokens so that the tokens of a block lie close together raises
 * their similarity). Host function: fills order[0 .. t*h*w) (host memory,
 * caller-owned) with the raster index (t-major, then h, then w) of the n-th
 * token along the curve; the curve is the Hilbert curve (Skilling's method)
 * of the smallest power-of-two cube holding the grid. Deterministic; needs no
 * GPU. SLA_ERR_INVALID_ARG for non-positive sides, more than 2^30 tokens or a
 * NULL order.
 */
SLA_API sla_status sla_hilbert_order(int32_t t, int32_t h, int32_t w, int32_t* order);

/*
 * Device gather / scatter of token rows (the reorder above, or any order).
 *   x, y    bf16 [rows, n_tok, d] device tensors, 16-byte aligned, not the same buffer
 *   order   int32 [n_order] device array, a permutation of 0 .. n_order-1
 *   inverse 0: y[r, n] = x[r, order[n]] for n < n_order;
 *           1: y[r, order[n]] = x[r, n] (undoes the gather)
 * Rows n >= n_order are copied in place. d must be a multiple of 8.
 * SLA_ERR_INVALID_ARG on bad pointers or sizes (nothing launched). An order
 * entry outside 0 .. n_order-1 is skipped on the device (no read or write for
 * it; the row it would have filled keeps its old contents).
 */
SLA_API sla_status sla_permute_tokens(const void* x, void* y, const int32_t* order, int32_t n_order,
                                      int32_t rows, int32_t n_tok, int32_t d, int32_t inverse,
                                      void* stream);

/*
 * Backward pass of the layer (fine-tuning with the layer in place:
 * SLA analysis page, arXiv 2509.24006, and SALAD summary, both train the model
 * with the sparse+linear layer for a few steps). The pages print no backward
 * pass; the gradients are those of L = sum(out * dout) with the routing held
 * fixed (the block classes are piecewise constant in the pooled scores and
 * carry no gradient):
 *   sparse branch   FlashAttention-style recomputation over the critical
 *                   blocks with the row log-sum-exp sla_forward kept in ws:
 *                   P = softmax rows, dP = dO V^T, dS = P * (dP - D_t),
 *                   D_t = dO_t . O_s,t; dQ = scale dS K, dK = scale dS^T Q,
 *                   dV = P^T dO (restricted to critical tiles)
 *   linear branch   u_t = phi(q_t) S'_i / (phi(q_t) . Z_i) with S'_i = S_i W_p,
 *                   du = g dO; dS'_i = sum_t phi(q_t)^T du_t / den_t,
 *                   dZ_i = -sum_t phi(q_t) (du_t . u_t) / den_t,
 *                   dh'_j = sum over rows i with j marginal of dS'_i (dz_j alike),
 *                   dphi(K_j) = (V_j W_p) dh'_j^T + dz_j, dV_j = phi(K_j) dh'_j W_p^T,
 *                   dW_p = sum_j V_j^T phi(K_j) dh'_j, chained through phi'
 *   gate            dg_t = dO_t . u_t, dlogit = dg g (1 - g): dq += dlogit w_g[h],
 *                   dw_g[h] += sum_t dlogit q_t
 *
 * Arguments:
 *   q, k, v, w_p, w_g, cfg  exactly as passed to the sla_forward call that
 *                           produced `out` (same values)
 *   out                     bf16 [B, H, N, d]: that call's output
 *   dout                    bf16 [B, H, N, d]: dL/dout (padding rows are ignored)
 *   dq                      bf16 [B, H, N, d]   written (padding rows 0)
 *   dk, dv                  bf16 [B, H_kv, N, d] written (padding rows 0)
 *   dw_p                    fp32, shape of w_p; written; may be NULL unless has_proj
 *   dw_g                    fp32 [H, d] ([H, 3, d] with nsa_branches); written; may
 *                           be NULL unless has_gate (the plain top-n mode has neither)
 *   ws                      the workspace of that sla_forward call, unchanged
 *                           since: the routing, the states S'_i, Z_i, phi(Q),
 *                           the gate and the row log-sum-exp are read from it
 *   bws                     device scratch of sla_backward_workspace_bytes(cfg)
 *                           bytes, 256-byte aligned; its first 256 bytes hold
 *                           this call's device status word (read it with
 *                           sla_check_device_status(bws, ...)). The flash
 *                           stages run persistent kernels (one CTA per SM) that
 *                           take their work units from counters in bws, zeroed
 *                           on `stream` before each launch: calls that share one
 *                           bws must not overlap on the GPU
 *   smooth-K        phi and phi' of k - m (m the head's mean valid key); every valid
 *                   row of dk also gets -1/N_valid times the head's summed
 *                   linear-branch gradient with respect to k - m
 *   top-n mode      the sparse branch only, over each query block's selected blocks and
 *                   window with the forward's element mask (s <= t, and block(s)
 *                   selected or s > t - window); dk, dv sum over the KV group's heads
 *   nsa_branches    O = sum_b g_b o_b over the compressed (b = 0), selected (1) and
 *                   window (2) branches, each its own softmax (sparse attention survey,
 *                   section 2, NSA). With e_b = dO_t . o_b,t each branch's attention
 *                   gradient is that of softmax attention with output gradient g_b dO;
 *                   the compressed keys and values are block means, so token s gets
 *                   1/cmp_block of the dK and dV of every compressed block that holds
 *                   it; with gates dlogit_b = e_b g_b (1 - g_b): dq += sum_b dlogit_b
 *                   w_g[h][b] and dw_g[h][b] += sum_t dlogit_b q_t. The forward call
 *                   keeps each branch's row log-sum-exp and output in ws for this.
 * Errors as for sla_forward. The parameter gradients are sums of per-block
 * partials added with floating-point atomics, so their last bits may vary from
 * run to run; dq, dk and dv are deterministic (NSA's compressed-key gradients are
 * summed from per-chunk partials in a fixed order).
 */
SLA_API size_t sla_backward_workspace_bytes(const sla_config* cfg);
SLA_API sla_status sla_backward(const void* q, const void* k, const void* v,
                                const void* w_p, const void* w_g, const sla_config* cfg,
                                const void* out, const void* dout,
                                void* dq, void* dk, void* dv, float* dw_p, float* dw_g,
                                const void* ws, size_t ws_bytes, void* bws, size_t bws_bytes,
                                void* stream);

/* Number of stages (kernel launches and memsets) sla_backward enqueues for cfg, or -1;
 * stage names as for the forward pass. */
SLA_API int32_t sla_backward_num_stages(const sla_config* cfg);
SLA_API const char* sla_backward_stage_name(const sla_config* cfg, int32_t s);

/* sla_backward with caller-created CUDA events around its stages, as sla_forward_timed. */
SLA_API sla_status sla_backward_timed(const void* q, const void* k, const void* v,
                                      const void* w_p, const void* w_g, const sla_config* cfg,
                                      const void* out, const void* dout,
                                      void* dq, void* dk, void* dv, float* dw_p, float* dw_g,
                                      const void* ws, size_t ws_bytes, void* bws, size_t bws_bytes,
                                      void* stream, void* const* events, int32_t n_events);

/* Static description of a status code. */
SLA_API const char* sla_status_string(sla_status s);

/* Library version, e.g. "0.1.0". */
SLA_API const char* sla_version(void);

/*
 * sla_route_noalloc - routing (steps 1-3) without a caller workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory on their call path: plugin hosts that hand a
 * library only its input and output buffers, code running under another
 * framework's memory pool that forbids allocations from outside it, and
 * latency-critical loops where a cudaMalloc / cudaFree (which may synchronise
 * the device) is not acceptable. Such callers cannot size and pass `ws`.
 *
 * Arguments, layouts and results are those of sla_route. The scratch that
 * sla_route keeps in `ws` (status word, pooled means, pooled scores) lives
 * instead in one static device array of SLA_NOALLOC_SCRATCH_BYTES (64 MiB),
 * which every GPU that loads the library holds until the process exits. The
 * call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine.
 *
 * - A configuration whose routing scratch exceeds SLA_NOALLOC_SCRATCH_BYTES is
 *   rejected with SLA_ERR_WORKSPACE before anything is launched (about 38 MB
 *   at B1 H12 N32768 d128; the scratch grows with B * H * (N / 64)^2).
 * - The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture. The
 *   address is cached per device together with the id of the CUDA context it
 *   belongs to; after a device reset (a new context) the next call looks it up
 *   again.
 * - All calls share the one array, which keeps the last call's contents (the
 *   status word is cleared at the start of every call). Calls that overlap on
 *   the GPU - on two streams, or from two host threads - race on it and must
 *   be serialised by the caller.
 */
#define SLA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
SLA_API sla_status sla_route_noalloc(const void* q, const void* k, const sla_config* cfg,
                                     int8_t* mask_out, int32_t* crit_idx, int32_t* neg_idx,
                                     void* stream);

/*
 * Device-side status of sla_route_noalloc (it has no caller workspace to hold
 * one). Synchronises `stream`, reads the status word at the start of the
 * current device's static routing array, clears it and returns what
 * sla_check_device_status returns for a workspace: SLA_OK, or
 * SLA_ERR_DEVICE_TIMEOUT / SLA_ERR_DEVICE_CHECK with *detail (nullable) naming
 * the kernel and check, or SLA_ERR_CUDA. Allocates nothing. Every
 * sla_route_noalloc call clears the word when it starts, so read it after the
 * call whose errors matter and before the next one.
 */
SLA_API sla_status sla_route_noalloc_status(void* stream, int32_t* detail);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H */
