/*
 * psa.h — C ABI of the B200 (sm_100a) Pyramid Sparse Attention forward pass.
 *
 * The method (arXiv:2512.04025, "PSA: Pyramid Sparse Attention for Efficient
 * Video Understanding and Generation", abstract): instead of keeping or
 * dropping whole KV blocks, each query block gives every KV block a pooling
 * level — the KV block itself (level 0) or its 2x / 4x / 8x average-pooled
 * form (levels 1..3) — or prunes it, and attends to the mixed-resolution keys
 * with one softmax.  The top168.com article on the paper names the three
 * components implemented here: pyramid KV construction by average pooling, a
 * multi-level mask generator driven by query-key block importance with
 * thresholds, and adaptive pyramid attention that keeps the probability
 * distribution consistent (here: each pooled key's logit gets + ln(c), c the
 * number of tokens it averages).
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    the library never allocates, frees or synchronises (psa_check_device is
 *    the one call that waits on the stream).  All work is enqueued on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - Tensors are dense row-major: Q/O [B, Hq, N, d], K/V [B, Hkv, N, d] with d
 *    contiguous; element type is params->dtype (fp32 or bf16).  Q, K, V and O
 *    must be 16-byte aligned; lse and block_mass, written one float at a
 *    time, 4-byte aligned; the workspace 256-byte aligned.
 *  - Arguments are validated on the host before anything is launched; on an
 *    error nothing is enqueued and a psa_status_t other than PSA_OK returns.
 *    A CUDA launch error is returned as PSA_ERR_CUDA.
 *  - Kernels never trap: a device wait that runs past its time limit sets an
 *    error word in the workspace and the kernel returns early; read it with
 *    psa_check_device (PSA_ERR_DEVICE_TIMEOUT).
 */
#ifndef PSA_H_
#define PSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PSA_OK = 0,
  PSA_ERR_INVALID_ARG = 1,          /* NULL pointer, bad size, tau not monotone, ... */
  PSA_ERR_UNSUPPORTED = 2,          /* valid but not implemented (e.g. d = 96)        */
  PSA_ERR_MISALIGNED = 3,           /* a device pointer breaks its alignment rule       */
  PSA_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace_bytes < psa_workspace_size(params)    */
  PSA_ERR_CUDA = 5,                 /* a CUDA call or launch failed                    */
  PSA_ERR_DEVICE_TIMEOUT = 6,       /* a kernel gave up waiting (see psa_check_device) */
  PSA_ERR_LEVEL_MAP = 7,            /* a caller's level map was corrected (see psa_attention_fwd) */
  PSA_ERR_DEVICE_BOUNDS = 8         /* debug builds: a work list failed its bounds check         */
} psa_status_t;

typedef enum { PSA_F32 = 0, PSA_BF16 = 1 } psa_dtype_t;

/* Level assignment rule (see psa_params_t.assign). */
typedef enum { PSA_ASSIGN_THRESHOLD = 0, PSA_ASSIGN_QUANTILE = 1 } psa_assign_t;

/* Problem description, shared by every entry point.
 *  B, Hq, Hkv, N, d  batch, query heads, KV heads (Hq % Hkv == 0; query head h
 *                    reads KV head h / (Hq / Hkv)), tokens, head dim (64 or 128).
 *  q_blk, kv_blk     query block (64 or 128) and KV block (64) sizes, in tokens.
 *  n_levels, pool    must be 4 and {1, 2, 4, 8}: level l pools 2^l tokens
 *                    ("Psa Pyramid Sparse Attention", Core Technique).
 *  tau               non-decreasing, in (0, 1].  With assign = PSA_ASSIGN_THRESHOLD
 *                    they are cumulative-mass thresholds: a KV block ranked r
 *                    gets the smallest level l with C_r < tau[l] (C_r = mass of
 *                    the blocks ranked before it), else it is pruned.  With
 *                    assign = PSA_ASSIGN_QUANTILE they are cumulative fractions
 *                    of the query block's visible KV blocks: the block ranked r
 *                    (0-based) gets the smallest l with r < K_l, K_l =
 *                    ceil(tau[l] * n_visible) computed exactly from the float
 *                    value, else it is pruned.  The level-assignment sketch of
 *                    "Psa Pyramid Sparse Attention" (Implementation: the top
 *                    int(n * keep_ratio) blocks at level 0, the rest in thirds,
 *                    nothing pruned) is the case K = (K_0, K_0 + r/3,
 *                    K_0 + 2r/3, n), r = n - K_0, with the thirds taken in rank
 *                    order (the sketch takes them in index order).
 *  causal            1: key position <= query position (blocks after the query
 *                    block are pruned, blocks straddling its diagonal get level
 *                    0 and a token mask).
 *  forced_prefix_tokens  visible KV blocks holding any of the first this-many
 *                    tokens get level 0 (e.g. a text prefix).
 *  scale             softmax scale; 0 means 1/sqrt(d).
 *  dtype             element type of Q, K, V, O and of the pooled levels.
 *  assign            level assignment rule (psa_assign_t): threshold on the
 *                    cumulative mass (the method's rule) or per-level quotas of
 *                    blocks by rank (the quantile-based rule the method is
 *                    compared with: top168.com article on PSA, ablations).
 *  sim_threshold     cosine-similarity constraint on the pyramid (the article's
 *                    ablations name such a constraint without defining it; this
 *                    is the library's reading).  Every pooled row of level
 *                    l >= 1 merges two rows of level l - 1; a merge is similar
 *                    when the cosine of its halves' mean keys is >=
 *                    sim_threshold (an empty or zero half passes).  A KV block
 *                    may use level l only when every merge at levels 1..l inside
 *                    it is similar; kept levels above that are lowered to it
 *                    (per KV head, after the overrides).  In [-1, 1]; -1 turns
 *                    the constraint off (every cosine passes), and so does any
 *                    value below -1.  NaN or a value above 1 is rejected.    */
typedef struct {
  int B, Hq, Hkv, N, d;
  int q_blk, kv_blk;
  int n_levels;
  int pool[4];
  float tau[4];
  int causal;
  int forced_prefix_tokens;
  float scale;
  psa_dtype_t dtype;
  psa_assign_t assign;
  float sim_threshold;
} psa_params_t;

/* Bytes of device workspace the calls below need for `params` (0 if params are
 * invalid).  The workspace holds: a device error word; pooled K/V levels 1..3
 * [B, Hkv, ceil(N/2^l), d] in dtype; level-3 keys in fp32 for scoring;
 * query-block means; block logits; an internal level map; the per-KV-block
 * largest level the cosine constraint allows; and the per-query-block work
 * list (KV block indices sorted by level, then index).  It is owned
 * by the caller and may be reused across calls with the same params. */
size_t psa_workspace_size(const psa_params_t* params);

/* Pyramid KV construction (top168.com article on PSA, pyramid paragraph and
 * component one: bottom level = original KV, each level up average-pooled).
 * K, V: device [B, Hkv, N, d].  Writes levels 1..3 of K and V and the fp32
 * level-3 keys into `workspace`.  Pooled row g of level l is the mean of tokens
 * [g*2^l, min((g+1)*2^l, N)), summed in fp32 and rounded once to dtype.
 * With sim_threshold > -1 it also records, per KV head and block, the largest
 * level the cosine-similarity constraint allows (cosines in fp32). */
psa_status_t psa_build_pyramid(const psa_params_t* params, const void* K, const void* V,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Multi-level mask generation (top168.com article, component two and the
 * threshold ablation; abstract of the paper: lower pooling levels for critical
 * KV blocks).  Needs the pyramid from psa_build_pyramid in `workspace`.
 * Q: device [B, Hq, N, d].  For each query block: q_bar = mean of its valid
 * rows (fp32); block logit z_j = logsumexp over block j's level-3 keys g of
 * (scale * q_bar . K3[g] + ln c_g); P = softmax over the visible blocks; rank
 * by P descending (ties to the lower j); level from tau as in psa_params_t;
 * then causal and forced-prefix overrides.  Writes the work list into
 * `workspace` and, if non-NULL:
 *   level_map  device int8 [B, Hq, ceil(N/q_blk), ceil(N/kv_blk)], -1 = pruned;
 *   block_mass device fp32, same shape: P (0 for blocks after a causal query block). */
psa_status_t psa_score_and_mask(const psa_params_t* params, const void* Q, void* workspace,
                                size_t workspace_bytes, int8_t* level_map, float* block_mass,
                                void* stream);

/* Adaptive pyramid attention (top168.com article, component three; the
 * paper's abstract: a kernel whose logical block size is decoupled from the
 * hardware tile).  Row i of query block a takes one softmax over every kept
 * key: for block j at level l = map[a][j] >= 0, block j's level-l pooled rows,
 * logit scale * q_i . K_l[g] + ln c_g.  Q, K, V: device, as above; K and V are
 * level 0 (the pyramid's other levels come from `workspace`).  level_map:
 * device int8 map to use instead of the one psa_score_and_mask built (NULL =
 * use the workspace's work list); a non-NULL map is turned into a work list
 * in `workspace` first, held to the contract the mask generator keeps: a
 * value outside -1..3 counts as pruned, and with causal = 1 a block after the
 * query block's last row is pruned and a kept block straddling its diagonal
 * is attended at level 0 with the token mask (a pooled key there would
 * average future tokens; the top168.com article's causal and bidirectional
 * paragraph has PSA serve causal generation).  The outputs are those of the
 * corrected map; if any entry had to be changed, the workspace error word
 * records it and the next psa_check_device returns PSA_ERR_LEVEL_MAP.
 * Nothing traps.  O: device [B, Hq, N, d] in dtype.  lse: device fp32
 * [B, Hq, N] natural-log sum of exp of the logits, or NULL.  A row that keeps
 * no key gets O = 0 and lse = -inf. */
psa_status_t psa_attention_fwd(const psa_params_t* params, const void* Q, const void* K,
                               const void* V, void* workspace, size_t workspace_bytes,
                               const int8_t* level_map, void* O, float* lse, void* stream);

/* The whole forward pass: psa_build_pyramid, psa_score_and_mask and
 * psa_attention_fwd in that order on one stream.  level_map (optional output,
 * device int8) receives the map that was used. */
psa_status_t psa_forward(const psa_params_t* params, const void* Q, const void* K, const void* V,
                         void* O, float* lse, int8_t* level_map, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Allocation-free forward pass.  The paper has no counterpart: this entry
 * point exists for callers that may not allocate device memory while they
 * run, such as a host framework that plans all memory ahead and hands a plugin
 * only its inputs and outputs, or a latency-sensitive loop that cannot afford
 * the device-wide synchronisation of cudaMalloc/cudaFree.  It does exactly
 * what psa_forward does, with the same arguments minus the workspace: the
 * scratch comes from a 32 MiB device array inside the library, held on every
 * GPU that loads the library until the process exits.
 *  - Returns PSA_ERR_WORKSPACE_TOO_SMALL, launching nothing, when
 *    psa_workspace_size(params) exceeds 32 MiB; invalid parameters give the
 *    same status as psa_forward.
 *  - Allocates nothing (no cudaMalloc/cudaFree); it clears the array's error
 *    word with cudaMemsetAsync on `stream`, then enqueues psa_forward's kernels.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call uses the same array, which keeps the previous call's contents:
 *    calls that overlap on the GPU (other streams, unordered host threads)
 *    race and give wrong results.  Serialise them.
 *  - A device timeout is recorded in the array's error word, which the next
 *    call clears; psa_check_device cannot read it. */
psa_status_t psa_forward_noalloc(const psa_params_t* params, const void* Q, const void* K,
                                 const void* V, void* O, float* lse, int8_t* level_map,
                                 void* stream);

/* psa_forward from host buffers, with the copies pipelined behind the
 * kernels: the heads are split into `head_groups` groups (contiguous query
 * heads with the KV heads they read: whole GQA groups when Hkv >= head_groups,
 * else an even split of each KV head's query heads, which needs head_groups a
 * multiple of Hkv), and for each batch element and group
 *   - the group's Q and not-yet-copied K, V go host -> device on h2d_stream,
 *   - the group's forward pass (psa_forward on the slices) runs on `stream`
 *     once they have arrived,
 *   - its O (and lse) go device -> host on d2h_stream,
 * so one group's copies overlap another's kernels.  Every (batch, head) is
 * independent, so the results equal one psa_forward over the whole problem.
 *  Q_host, K_host, V_host, O_host, lse_host: host memory in the layout of
 *    psa_forward (pinned memory lets the copies run asynchronously).
 *  Q_dev, K_dev, V_dev, O_dev, lse_dev: device buffers for the whole problem,
 *    aligned as for psa_forward; lse_host and lse_dev are both NULL or both
 *    set.
 *  workspace: psa_workspace_size(params) bytes (groups reuse it in turn).
 *  stream, h2d_stream, d2h_stream: three distinct streams; everything is
 *    enqueued, and `stream` completes only after the last copy to the host.
 * Returns PSA_ERR_INVALID_ARG for bad parameters, a NULL buffer, streams that
 * are not distinct or a group split that cannot be made; otherwise the status
 * of the copies and of psa_forward. */
psa_status_t psa_forward_host(const psa_params_t* params, const void* Q_host, const void* K_host,
                              const void* V_host, void* O_host, float* lse_host, void* Q_dev,
                              void* K_dev, void* V_dev, void* O_dev, float* lse_dev,
                              void* workspace, size_t workspace_bytes, int head_groups,
                              void* stream, void* h2d_stream, void* d2h_stream);

/* Bytes of the scratch psa_backward needs besides the forward workspace (the
 * per-row D = dO . O and the fp32 gradients of every pyramid level), or 0 if
 * params is invalid. */
size_t psa_backward_workspace_size(const psa_params_t* params);

/* Gradient of the pyramid attention with the level map held fixed: dQ, dK,
 * dV of the forward pass's O with respect to Q, K and V, given dO.
 * Source: adaptive pyramid attention (top168.com article on PSA, component
 * three) differentiated by the chain rule.  The map is a discrete function of
 * Q and K and passes no gradient; the ln c logit bias is a constant.  With
 * P_ig = exp(s q_i . K_l[g] + ln c_g - lse_i) over row i's kept keys,
 * D_i = dO_i . O_i and dX_ig = P_ig (dO_i . V_l[g] - D_i):
 *   dQ_i = s sum_g dX_ig K_l[g],
 *   dK_l[g] = s sum_i dX_ig q_i,  dV_l[g] = sum_i P_ig dO_i,
 * and each pooled row's gradient, divided by its token count c_g, goes to
 * each of the c_g tokens it averages.  A KV head's gradients sum over the
 * query heads that read it.  Rows that kept no key pass no gradient.
 *  Q, K, V, O, dO: device, layouts of psa_forward; O and lse are the forward
 *    pass's outputs for the same inputs and map.
 *  lse: device fp32 [B, Hq, N], natural log, required.
 *  level_map: device int8 [B, Hq, Nq, Nk] or NULL.  NULL: the work list the
 *    last forward call left in `workspace` is used (so call this after
 *    psa_forward / psa_attention_fwd with the same workspace); else the list
 *    is rebuilt from the map, as psa_attention_fwd does (with the same
 *    corrections and PSA_ERR_LEVEL_MAP report).
 *  workspace: the forward workspace, psa_workspace_size(params) bytes; the
 *    pyramid levels in it are rebuilt from K and V.
 *  bwd_workspace: device, 256-byte aligned, psa_backward_workspace_size(params)
 *    bytes; caller-owned scratch, overwritten.
 *  dQ [B, Hq, N, d], dK, dV [B, Hkv, N, d]: device outputs in the input dtype,
 *    16-byte aligned; every element is written.
 * dQ is deterministic.  dK and dV are summed in fp32 with atomic adds (a pooled
 * row collects from every query block that keeps it), whose order varies, so
 * repeated calls agree to rounding, not bit for bit.
 * Asynchronous on `stream`.  Errors as psa_forward (PSA_ERR_INVALID_ARG for a
 * NULL lse or bwd_workspace). */
psa_status_t psa_backward(const psa_params_t* params, const void* Q, const void* K, const void* V,
                          const void* O, const float* lse, const void* dO,
                          const int8_t* level_map, void* workspace, size_t workspace_bytes,
                          void* bwd_workspace, size_t bwd_workspace_bytes, void* dQ, void* dK,
                          void* dV, void* stream);

/* Waits for `stream`, then reads and clears the workspace's device error word.
 * Returns PSA_ERR_DEVICE_TIMEOUT if a kernel gave up waiting since the last
 * check, else PSA_ERR_DEVICE_BOUNDS if (debug builds) a work list failed its
 * bounds check, else PSA_ERR_LEVEL_MAP if a caller's level map was corrected
 * (psa_attention_fwd, psa_backward), PSA_ERR_CUDA if the stream reported an
 * error, else PSA_OK. */
psa_status_t psa_check_device(const psa_params_t* params, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Failure-path self-test; the method has no counterpart.  Enqueues on
 * `stream` one warp that waits, through the same bounded-wait code as the
 * tensor-core kernels, on a barrier that nothing ever arrives at, and gives
 * up after `limit_ns` nanoseconds (1 ns .. 1 s), recording a timeout in the
 * workspace's device error word exactly as a kernel that timed out would.
 * The next psa_check_device then returns PSA_ERR_DEVICE_TIMEOUT (and clears
 * the word).  Nothing faults or traps.  params: any valid description whose
 * workspace layout `workspace` holds; workspace: device, 256-byte aligned, at
 * least psa_workspace_size(params) bytes (PSA_ERR_WORKSPACE_TOO_SMALL,
 * PSA_ERR_MISALIGNED otherwise).  Returns PSA_ERR_INVALID_ARG for a null
 * argument or a limit outside 1 ns .. 1 s, PSA_ERR_CUDA for a launch error. */
psa_status_t psa_selftest_wait_timeout(const psa_params_t* params, void* workspace,
                                       size_t workspace_bytes, uint64_t limit_ns, void* stream);

/* 1 when the library was compiled with PSA_DEBUG (libpsa_debug.so), else 0;
 * the method has no counterpart.  A debug build checks, on the device, every
 * work list in the workspace before the attention kernels (forward and
 * backward) walk it: a query block whose level counts are negative or add up
 * to more than ceil(N / kv_blk), or whose entries leave that range or are not
 * increasing inside a level, is skipped (O = 0, lse = -inf, no gradient) and
 * recorded in the error word, which psa_check_device reports as
 * PSA_ERR_DEVICE_BOUNDS.  Lists written by this library always pass; the
 * check guards against a workspace corrupted between calls.  Nothing traps. */
int psa_debug_build(void);

/* Static description of a status code. */
const char* psa_status_string(psa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* PSA_H_ */
