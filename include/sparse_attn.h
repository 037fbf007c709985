/*
 * sparse_attn.h -- C ABI of libsparse_attn.so: top-k index-selected sparse
 * attention (forward and backward) on one NVIDIA B200 (sm_100a).
 *
 * The operation.  For every query token t and kv-head g, a set of KV rows is
 * selected and attended to by the G = Hq / Hkv query heads that share g:
 *
 *   - block-level selection: aclnnSparseFlashAttentionGrad, "Formula" --
 *     selectedKey = Gather(key, topkIndices[i]), 0 <= i < selectBlockCount,
 *     each index naming block_size contiguous rows;
 *   - token-level selection of a shared latent KV (K = V) and the sliding
 *     window / compressed-KV concatenation: SparseFlashMlaGrad, "Computation
 *     formula", Stage 1, with the oriSparseIndices / cmpSparseIndices,
 *     oriTopkLength / cmpTopkLength, oriMaskMode / cmpMaskMode, oriWinLeft /
 *     oriWinRight and sinks rows of its "Parameter Description" table;
 *   - forward: aclnnNsaSelectedAttentionInfer, "Formula" --
 *     O = Softmax(Q K_sel^T * scale) V_sel, lse = ln(sum exp(scores) [+ exp(sink)]);
 *   - backward: SparseFlashMlaGrad, "Computation formula", Stages 2-3, and
 *     aclnnSparseFlashAttentionGrad, "Formula", Phases 1-3 --
 *     P = exp(S - lse), dP = dO V^T, dS = P o (dP - rowsum(dO o O)),
 *     dQ = dS K scale, dK = dS^T Q scale, dV = P^T dO (dKV = dK + dV when K = V),
 *     dSinks = sum over rows of -P_sink * sum_j P_j dP_j.
 *
 * Call shape.  Like the pages' two-phase API: *_get_workspace_size validates
 * the arguments on the host and returns the workspace the call needs; the
 * second call re-validates, enqueues its kernels on the caller's stream and
 * returns without synchronising.  The library never allocates device memory:
 * the caller owns every buffer, including the workspace.
 *
 * Pointers.  Every tensor pointer is a DEVICE pointer (row-major, innermost
 * dimension contiguous, 16-byte aligned).  "bf16" below means the 2-byte element
 * type sa_args.dtype names: bfloat16 (SA_DTYPE_BF16) or IEEE half
 * (SA_DTYPE_FP16), the same for q, k, v, kv, cmp_kv, O, dO and the gradients
 * (SparseFlashMlaGrad "Parameter Description": BFLOAT16 or FLOAT16, outputs of
 * the inputs' type); lse, sinks, dSinks and the SoftmaxL1Norm outputs are fp32.
 * The tensor-core kernels take bfloat16; fp16 problems run on the generic
 * query-stationary kernels (fp16 MMA operands, fp32 accumulation), whatever the
 * selection mode.  The sa_args /
 * sa_fwd_out / sa_bwd_io structs themselves are host memory read during the
 * call only.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *
 * Layouts (layout_q for q / o / d_o / lse / the index tensors, layout_kv for
 * k / v / kv / cmp_kv, each SA_LAYOUT_BSND or SA_LAYOUT_TND, as the pages'
 * layoutQ / layoutKv rows; only equal layouts are built, a mix returns
 * SA_ERR_UNSUPPORTED):
 *   BSND: q [B, s_q, Hq, d_qk]   k [B, s_kv, Hkv, d_qk]   v [B, s_kv, Hkv, d_v]
 *         kv [B, s_kv, Hkv, d_qk] (K = V)  cmp_kv [B, s_kv / cmp_ratio, Hkv, d_qk]
 *         ori_idx [B, s_q, Hkv, topk]  cmp_idx [B, s_q, Hkv, cmp_topk]
 *         ori_topk_len / cmp_topk_len [B, s_q, Hkv]
 *         o / d_o [B, s_q, Hq, d_v]   lse [B, s_q, Hq] (fp32)
 *   TND:  the same with the leading [B, s] replaced by a packed token axis:
 *         q [t_q, ...], k / v / kv [t_kv, ...], cmp_kv [t_cmp, ...]; sequence b
 *         spans [cu_seqlens_x[b], cu_seqlens_x[b+1]) (B + 1 int32 offsets).
 * Index values are positions local to their own sequence: a block index x
 * covers rows [x * block_size, (x + 1) * block_size) clipped to the sequence;
 * a token / compressed index is one row.  A negative index, or a slot at or
 * past the row's topk length, selects nothing.  Indices past the end of the
 * sequence are never read: they select nothing, and with SA_FLAG_CHECK the
 * call reports SA_ERR_INDEX.
 *
 * Masks (applied per query row t, aligned bottom-right: ta = t + len_kv - len_q):
 *   ori: NONE; CAUSAL row r <= ta; BAND ta - ori_win_left <= r <= ta + ori_win_right.
 *   cmp: NONE; CAUSAL compressed row c visible iff (c + 1) * cmp_ratio - 1 <= ta.
 * Without ori indices the whole original KV enters the selection under the ori
 * mask (sliding window when BAND); cmp indices add compressed rows (SCFA); a
 * compressed KV without indices adds all its rows under the cmp mask (CFA).
 *
 * Paged KV cache (aclnnNsaSelectedAttentionInfer: "paged attention obtains the
 * kvCache", a few query tokens per sequence).  With block_table, k / v / kv are a
 * cache of t_kv rows in pages of page_size rows; logical row r of sequence b is
 * cache row block_table[b, r / page_size] * page_size + r % page_size.  s_kv is the
 * logical capacity (at most max_pages * page_size) and seqused_kv gives each
 * sequence's actual length; the queries sit at the end of their sequences (the
 * bottom-right alignment).  BSND only, no compressed KV; the forward and
 * sa_softmax_l1norm take it, the backward returns SA_ERR_UNSUPPORTED.  A page
 * index outside the cache selects nothing and raises the index bit.
 *
 * Used lengths (SparseFlashMlaGrad "Parameter Description": sequsedQOptional,
 * sequsedOriKvOptional, sequsedCmpKvOptional).  When given, sequence b takes part
 * with its first seqused_q[b] query tokens, seqused_kv[b] KV rows and
 * seqused_cmp[b] compressed rows (each clamped to the sequence's length): these
 * effective lengths set the bottom-right alignment (ta = t + used_kv - used_q) and
 * the sequence ends, an index past them selects nothing, and a query row past
 * seqused_q is an empty row (below).  Problems with used lengths run on the
 * generic and token-level kernels.
 *
 * Empty rows.  A query row with no visible key and no sink gets lse = +inf and
 * O = 0 and contributes no gradient.  A call with no query tokens returns
 * SA_OK without launching anything.
 *
 * Determinism.  The backward accumulates dK / dV / dKV / dSinks with fp32
 * atomics, so results may differ in the last bits from run to run.
 *
 * Streams.  Calls only enqueue kernels and memsets on the caller's stream, so
 * they capture into CUDA graphs.  The backward's kernels are launched with
 * programmatic dependent launch: each may start its shared-memory and TMEM
 * set-up while the kernel before it on the stream finishes, and waits for that
 * kernel's completion before it reads or writes global memory, so stream
 * order is kept for the caller's own work before and after the call.
 *
 * Status word.  The first 4 bytes of every forward or backward workspace are a
 * status word that each call clears before its kernels run and that the
 * kernels OR bits into:
 *   1  an index past the end of its sequence was met (it selected nothing);
 *   2  a bounded device wait gave up (the call's outputs are incomplete);
 *   4  a kernel found its shared memory misaligned and did nothing.
 * sa_read_status() synchronises the stream and maps the word to SA_OK,
 * SA_ERR_TIMEOUT (bit 2), SA_ERR_INDEX (bit 1) or SA_ERR_CUDA (bit 4).
 *
 * Bounded waits.  The tensor-core kernels' waits give up after about two
 * seconds; the kernel then raises the timeout bit in the status word and
 * finishes without completing its work (see sa_selftest_wait_timeout).
 *
 * Errors.  Every entry point returns an sa_status.  Argument errors are found
 * on the host before anything is enqueued.  CUDA launch errors come back as
 * SA_ERR_CUDA (the library calls cudaGetLastError after its launches).
 * Device-side conditions (timeouts, out-of-range indices) are read back with
 * sa_read_status(), or at once with SA_FLAG_CHECK for indices.
 */
#ifndef SPARSE_ATTN_H_
#define SPARSE_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SA_ABI_VERSION 4

typedef enum sa_status {
  SA_OK = 0,
  SA_ERR_NULLPTR = 1,      /* a required pointer is NULL */
  SA_ERR_PARAM = 2,        /* a size, mode or attribute is out of range */
  SA_ERR_UNSUPPORTED = 3,  /* valid per the pages but not built (e.g. mixed layouts) */
  SA_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than *_get_workspace_size */
  SA_ERR_INDEX = 5,        /* SA_FLAG_CHECK found an index past its sequence */
  SA_ERR_TIMEOUT = 6,      /* a bounded device wait gave up */
  SA_ERR_CUDA = 7          /* a CUDA runtime error */
} sa_status;

typedef enum sa_layout { SA_LAYOUT_BSND = 0, SA_LAYOUT_TND = 1 } sa_layout;
typedef enum sa_mask { SA_MASK_NONE = 0, SA_MASK_CAUSAL = 1, SA_MASK_BAND = 2 } sa_mask;
typedef enum sa_dtype { SA_DTYPE_BF16 = 0, SA_DTYPE_FP16 = 1 } sa_dtype;

/* flags */
#define SA_FLAG_CHECK 1u   /* validate every index on the device first; the call then
                              synchronises `stream` and returns SA_ERR_INDEX if one is
                              past its sequence (nothing else is computed) */
/* Backward kernel choice (results agree within rounding; the default is the
 * fastest measured; sa_plan() reports which kernel a problem gets).
 * Block-level selection with block_size 64, BSND, equal query / key lengths,
 * separate K and V and no sinks runs key-stationary by default: one CTA per
 * (kv block, chunk of the tokens that select it) accumulates dK / dV on the
 * tensor cores and adds its dQ contributions to an fp32 accumulator with
 * vector atomics (Tq*Hq*d_qk*4 workspace bytes).  Token-level selection over
 * one shared KV row of 576 (V = its first 512 columns) with a multiple of 64
 * query heads per kv-head runs the tensor-core token kernel.  Every other
 * problem runs the generic query-stationary kernel. */
#define SA_FLAG_QUERY_STATIONARY_BWD 2u  /* force the generic query-stationary backward
                                            (dK / dV by fp32 scatter-add) */
#define SA_FLAG_DQ_SEPARATE 4u  /* key-stationary backward: take dQ from a separate
                                   query-stationary pass instead of atomics; honoured
                                   only when topk <= 256 (otherwise ignored) */
/* Forward kernel choice for block-level selection (64-row blocks, BSND, equal
 * lengths, separate K and V, no sinks, topk <= 256).  The default is the
 * TMA-fed query-stationary kernel with mma.sync tiles: that forward is bound by
 * gathering the selected blocks from L2 (every 16-head item streams its blocks'
 * K and V once), which the warp-level MMAs keep up with.  This flag selects the
 * tcgen05 version instead (scores and output in TMEM, M = 128 key pairs against
 * the 16 heads of an item); it computes the same result and measured slower. */
#define SA_FLAG_FWD_BLOCK_TC 8u
/* Token-level tensor-core forward: with a multiple of 128 query heads per kv-head
 * the two 64-head CTAs of a token run as a thread-block cluster and share the row
 * gathers (each gathers every other 32-row sub-tile and copies it to the other
 * over distributed shared memory).  This flag runs every 64-head CTA on its own
 * instead; the result is bit-identical.  It also serves where a two-CTA cluster of
 * this kernel's shared memory cannot be scheduled (the launch then fails and
 * sa_fwd returns SA_ERR_CUDA): the unpaired kernel needs no clusters. */
#define SA_FLAG_TOKEN_FWD_UNPAIRED 16u

/* Kernels reported by sa_plan(). */
typedef enum sa_kernel {
  SA_KERNEL_FWD_BLOCK = 1,         /* forward, query-stationary over 64-row blocks (topk <= 256),
                                      TMA-fed, mma.sync tiles */
  SA_KERNEL_FWD_TOKEN_TC = 2,      /* forward, token-level shared KV 576/512 on tcgen05 */
  SA_KERNEL_FWD_GENERIC = 3,       /* forward, any selection, rows gathered one by one */
  SA_KERNEL_BWD_KEY_STATIONARY = 4,        /* backward, key-stationary, dQ by atomics */
  SA_KERNEL_BWD_KEY_STATIONARY_DQ_PASS = 5,/* backward, key-stationary + separate dQ pass */
  SA_KERNEL_BWD_TOKEN_TC = 6,      /* backward, token-level shared KV 576/512 on tcgen05 */
  SA_KERNEL_BWD_GENERIC = 7,       /* backward, any selection, dK / dV by fp32 scatter-add */
  SA_KERNEL_FWD_BLOCK_TC = 8       /* forward, the same block problems on tcgen05 (SA_FLAG_FWD_BLOCK_TC) */
} sa_kernel;

/* Views of sa_debug_block_index(). */
#define SA_INDEX_VIEW_QUERY_BLOCKS 0  /* usable slots as the query-stationary block kernels see them */
#define SA_INDEX_VIEW_KEY_LISTS 1     /* the key-stationary backward's inverse index */

/* The problem description shared by every entry point (host struct). */
typedef struct sa_args {
  int32_t layout_q;        /* sa_layout of q, o, d_o, lse and the index tensors */
  int32_t layout_kv;       /* sa_layout of k, v, kv and cmp_kv (must equal layout_q) */
  int32_t dtype;           /* sa_dtype: the 2-byte element type of every bf16 tensor */
  int32_t batch;           /* B >= 0 */
  int32_t s_q, s_kv;       /* BSND sequence lengths (ignored for TND) */
  int32_t t_q, t_kv, t_cmp;/* TND packed token counts (ignored for BSND) */
  int32_t n_heads_q;       /* Hq, a multiple of n_heads_kv */
  int32_t n_heads_kv;      /* Hkv */
  int32_t d_qk;            /* score head dim; multiple of 16, <= 576 */
  int32_t d_v;             /* value head dim; multiple of 16, <= 512; <= d_qk if kv_shared */
  int32_t kv_shared;       /* 1: K = V = kv, V is the first d_v columns of each kv row */
  int32_t block_size;      /* rows per ori index (1 = token-level); <= 64 or a multiple of 64 */
  int32_t topk;            /* ori index slots per (token, kv-head); 0 = no ori indices */
  int32_t cmp_topk;        /* cmp index slots per (token, kv-head); 0 = no cmp indices (then cmp_kv,
                              when given with cmp_ratio > 1, contributes all its rows: CFA) */
  int32_t cmp_ratio;       /* >= 1; cmp_kv has len_kv / cmp_ratio rows per sequence */
  int32_t ori_mask_mode;   /* sa_mask */
  int32_t cmp_mask_mode;   /* SA_MASK_NONE or SA_MASK_CAUSAL */
  int64_t ori_win_left;    /* BAND: past rows kept (>= 0) */
  int64_t ori_win_right;   /* BAND: future rows kept (>= 0) */
  float scale;             /* scaleValue: multiplies Q K^T */
  uint32_t flags;          /* SA_FLAG_* */
  const void* q;           /* bf16, required */
  const void* k;           /* bf16, required when !kv_shared */
  const void* v;           /* bf16, required when !kv_shared */
  const void* kv;          /* bf16, required when kv_shared */
  const void* cmp_kv;      /* bf16, required when cmp_topk > 0; without cmp indices and with
                              cmp_ratio > 1 every compressed row takes part (CFA) */
  const int32_t* ori_idx;  /* required when topk > 0 */
  const int32_t* cmp_idx;  /* required when cmp_topk > 0 */
  const int32_t* cu_seqlens_q;   /* TND: B + 1 offsets, required */
  const int32_t* cu_seqlens_kv;  /* TND: B + 1 offsets, required */
  const int32_t* cu_seqlens_cmp; /* TND with a compressed KV: B + 1 offsets, required */
  const int32_t* ori_topk_len;   /* optional (NULL = all topk slots usable) */
  const int32_t* cmp_topk_len;   /* optional (NULL = all cmp_topk slots usable) */
  const int32_t* cmp_residual;   /* optional, [B]: len_kv mod cmp_ratio; accepted, not used */
  const float* sinks;            /* optional, [Hq] fp32 sink logits */
  const int32_t* seqused_q;      /* optional, [B]: query tokens of each sequence that take part
                                    (sequsedQ); the rest select nothing */
  const int32_t* seqused_kv;     /* optional, [B]: original KV tokens of each sequence that take
                                    part (sequsedOriKv) */
  const int32_t* seqused_cmp;    /* optional, [B]: compressed KV rows of each sequence that take
                                    part (sequsedCmpKv) */
  const int32_t* block_table;    /* optional, [B, max_pages]: paged KV cache (BSND only) */
  int32_t page_size;             /* rows per cache page (with block_table) */
  int32_t max_pages;             /* pages per sequence in block_table (with block_table) */
} sa_args;

/* Forward outputs (device): O bf16 [.., Hq, d_v]; lse fp32 [.., Hq]. */
typedef struct sa_fwd_out {
  void* o;
  float* lse;
} sa_fwd_out;

/* Backward inputs and outputs (device).  o / lse are the forward's outputs.
 * dq is required.  dk and dv (separate K, V) or dkv (K = V) are required.
 * dcmp_kv is required with a compressed KV (cmp indices, or CFA), dsinks when sinks != NULL. */
typedef struct sa_bwd_io {
  const void* o;           /* bf16 [.., Hq, d_v] */
  const void* d_o;         /* bf16 [.., Hq, d_v] */
  const float* lse;        /* fp32 [.., Hq] */
  void* dq;                /* bf16, shape of q */
  void* dk;                /* bf16, shape of k */
  void* dv;                /* bf16, shape of v */
  void* dkv;               /* bf16, shape of kv */
  void* dcmp_kv;           /* bf16, shape of cmp_kv */
  float* dsinks;           /* fp32 [Hq] */
} sa_bwd_io;

/* ---- forward ---------------------------------------------------------- */

/* Phase 1: validate `args` (host only) and return the forward workspace size. */
sa_status sa_fwd_get_workspace_size(const sa_args* args, size_t* ws_bytes);

/* Phase 2: compute O and lse.  `ws` must hold at least the phase-1 size
 * (may be NULL when that size is 0).  Enqueued on `stream`, asynchronous. */
sa_status sa_fwd(const sa_args* args, const sa_fwd_out* out, void* ws, size_t ws_bytes,
                 void* stream);

/* ---- backward --------------------------------------------------------- */

/* Phase 1: validate `args` (host only) and return the backward workspace size
 * (fp32 accumulators for dK/dV, dKV and dCmpKv, the rowsum(dO o O) vector and
 * the inverse index used by the key-stationary kernels). */
sa_status sa_bwd_get_workspace_size(const sa_args* args, size_t* ws_bytes);

/* Phase 2: compute dQ, dK/dV (or dKV), dCmpKv and dSinks from dO, O and lse.
 * Every output is fully overwritten.  Enqueued on `stream`, asynchronous. */
sa_status sa_bwd(const sa_args* args, const sa_bwd_io* io, void* ws, size_t ws_bytes,
                 void* stream);

/* The backward pass for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry point.  Some callers cannot call
 * cudaMalloc where they run the backward: a plugin whose host framework owns
 * all device memory through its own pre-reserved pool and forbids allocation
 * during execution, or a latency-critical loop that cannot absorb the device
 * synchronisation an allocation implies.  This entry point needs no
 * workspace: it runs sa_bwd on a fixed scratch array compiled into the
 * library (sa_bwd_no_alloc_max_workspace() bytes, held on every GPU that loads
 * the library until the process exits) and allocates nothing.
 *   - Problems whose sa_bwd_get_workspace_size exceeds that size are rejected
 *     with SA_ERR_WORKSPACE before anything is enqueued.
 *   - The first call in a CUDA context (the device's primary context, with
 *     that device current) resolves the array's device address once; make
 *     that first call before any stream capture.  A new context on the same
 *     device (after cudaDeviceReset, or one made current through the driver
 *     API) resolves it again.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (other streams, other host threads on the same device) race.  Each call
 *     re-zeroes the parts it uses, so nothing carries over between calls.
 * Inputs, outputs and errors are as for sa_bwd.  Asynchronous. */
sa_status sa_bwd_no_alloc(const sa_args* args, const sa_bwd_io* io, void* stream);

/* Size in bytes of the scratch array behind sa_bwd_no_alloc. */
size_t sa_bwd_no_alloc_max_workspace(void);

/* The SoftmaxL1Norm outputs of SparseFlashMlaGrad ("Parameter Description":
 * oriSoftmaxL1NormOptional, cmpSoftmaxL1NormOptional, FLOAT32): the target
 * distribution of the indexer loss (aclnnSparseLightningIndexerGradKLLoss,
 * "Formula": the attention scores summed over all heads, then L1-normalised along
 * the context).  With P = exp(scale q.k - lse), the softmax the backward
 * recomputes (sink included in lse; the sink is no slot):
 *   ori_out[token, kv-head, s] = sum over the kv-head's query heads and over the
 *                                visible rows of ori slot s of P, divided by the
 *                                sum of that row over all its ori slots;
 *   cmp_out likewise over the cmp slots (each output is normalised on its own).
 * Empty slots (index < 0, slot >= the topk length, no visible row) hold 0; a row
 * with no visible slot is all 0.  An index past its sequence selects nothing.
 * lse fp32 [.., Hq] from sa_fwd (device).  ori_out fp32 [.., Hkv, topk] (needs ori
 * indices: topk > 0) and cmp_out fp32 [.., Hkv, cmp_topk] (needs cmp indices), both
 * device buffers the call overwrites; either may be NULL, not both.  Needs no
 * workspace.  Errors: SA_ERR_NULLPTR (no output, or no lse), SA_ERR_PARAM (an
 * output without its index list, misaligned tensors), validation errors as for
 * sa_fwd.  Asynchronous. */
sa_status sa_softmax_l1norm(const sa_args* args, const float* lse, float* ori_out, float* cmp_out, void* stream);

/* The lightning indexer's KL-loss backward (aclnnSparseLightningIndexerGradKLLoss,
 * "Formula"): over token t's used slots j (index >= 0, before topk_len, inside the
 * sequence, not in t's future),
 *   I[t, j] = sum_h w[t, h] ReLU(q[t, h] . k[j]),  L = sum_t KL(p[t, :] || Softmax(I[t, :])),
 *   dI = Softmax(I) - p,  dw[t, h] = sum_j ReLU(q[t, h] . k[j]) dI[t, j],
 *   dS = w[t, h] (q[t, h] . k[j] > 0) dI[t, j],  dq[t] = dS k,  dk[j] += dS^T q[t].
 * p's entries at unused slots are ignored; 0 log 0 = 0; no scale on q k^T. */
typedef struct sa_indexer_args {
  int32_t layout;          /* sa_layout of every tensor (BSND or TND) */
  int32_t batch;           /* B */
  int32_t s_q, s_kv;       /* BSND sequence lengths */
  int32_t t_q, t_kv;       /* TND packed token counts */
  int32_t n_heads;         /* indexer query heads H: 16, 32 or 64 */
  int32_t d;               /* head dim: 64 or 128 */
  int32_t topk;            /* index slots per token (>= 1) */
  const void* q;           /* bf16 [.., H, d] */
  const void* k;           /* bf16 [.., d] (one indexer key head) */
  const float* w;          /* fp32 [.., H] per-token head weights */
  const int32_t* idx;      /* [.., topk] token indices local to the sequence, -1 = empty */
  const int32_t* topk_len; /* optional [..]: usable slots per token */
  const float* p;          /* fp32 [.., topk] target distribution (e.g. sa_softmax_l1norm's ori_out) */
  const int32_t* cu_seqlens_q;   /* TND: B + 1 offsets */
  const int32_t* cu_seqlens_kv;  /* TND: B + 1 offsets */
} sa_indexer_args;

typedef struct sa_indexer_grads {
  float* loss;             /* optional, fp32 [..]: each token's KL term */
  void* dq;                /* bf16 [.., H, d] */
  void* dk;                /* bf16 [.., d] */
  float* dw;               /* fp32 [.., H] */
} sa_indexer_grads;

/* Workspace of sa_indexer_kl_grad: a status word and the fp32 dk accumulator. */
sa_status sa_indexer_kl_grad_get_workspace_size(const sa_indexer_args* args, size_t* ws_bytes);
/* Errors: SA_ERR_NULLPTR (a required pointer), SA_ERR_PARAM (sizes, alignment),
 * SA_ERR_UNSUPPORTED (H or d not built), SA_ERR_WORKSPACE.  Asynchronous; an index
 * past its sequence sets the status word's index bit (sa_read_status). */
sa_status sa_indexer_kl_grad(const sa_indexer_args* args, const sa_indexer_grads* grads, void* ws,
                             size_t ws_bytes, void* stream);

/* rowsum(dO o O) alone -- the "FlashSoftmaxGrad(dO, O)" / "SoftmaxGrad(dO, O)"
 * term of aclnnSparseFlashAttentionGrad Phase 2 and SparseFlashMlaGrad Stage 2:
 * delta[token, h] = sum_c d_o[token, h, c] * o[token, h, c] in fp32.
 * o, d_o bf16 [.., Hq, d_v]; delta fp32 [.., Hq] (device).  Asynchronous. */
sa_status sa_softmax_grad_preprocess(const sa_args* args, const void* o, const void* d_o,
                                     float* delta, void* stream);

/* ---- inspection ------------------------------------------------------- */

/* The visible KV set of every (query token, kv-head) unit exactly as the
 * kernels resolve it (Stage 1 selection plus masks).  rows: int32
 * [units, max_rows] with unit = token * Hkv + g; original-KV row r is written
 * as r, compressed row c as (0x40000000 | c), in slot order; entries past the
 * count are left untouched.  counts: int32 [units], the full count (may exceed
 * max_rows, in which case only max_rows entries are written).  Asynchronous. */
sa_status sa_debug_resolve(const sa_args* args, int32_t* rows, int32_t* counts,
                           int32_t max_rows, void* stream);

/* ---- benchmarking hooks ------------------------------------------------ */

/* Timing hook (process-wide, not thread-safe): when both events are
 * non-NULL, later sa_fwd / sa_bwd calls record ev_begin right before and
 * ev_end right after one of their kernels, on the call's stream:
 *   which = 0: the forward kernel;
 *   which = 1: the backward kernel that forms dK / dV (key-stationary kernel,
 *              or the fused query-stationary kernel);
 *   which = 2: the query-stationary dQ pass of the key-stationary backward.
 * Both are cudaEvent_t created by the caller; pass NULL, NULL to disable. */
void sa_set_timing_events(void* ev_begin, void* ev_end, int32_t which);

/* Number of kernels this library has launched since it was loaded
 * (memsets excluded). */
int64_t sa_kernel_launch_count(void);

/* Self-check of the tensor-core building blocks used by the key-stationary
 * backward: one CTA computes D = A B with TMA loads (boxes of box_rows x 64),
 * 128-byte swizzled shared-memory operands, tcgen05.mma and TMEM loads.
 * A is K-major [M][K] (a_mn = 0) or MN-major [K][M] (a_mn = 1); B is K-major
 * [N][K] (b_mn = 0) or MN-major [K][N] (b_mn = 1); all bf16 row-major, device.
 * D fp32 [M][N] (device).  M in {64, 128}; N, K multiples of 64, N <= 256,
 * K <= 256; box_rows in {8, 16, 32, 64}.  d_lane: TMEM lane offset of the
 * accumulator, 0, or 16 with M = 64 (an M = 64 accumulator occupies 16 lanes of
 * each 32-lane sub-partition, so two of them can share columns).  *status
 * (device int) gets the timeout bit if a bounded wait gives up.  Asynchronous. */
sa_status sa_selftest_mma(int32_t M, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn, int32_t box_rows,
                          int32_t d_lane, const void* A, const void* B, float* D, int32_t* status,
                          void* stream);

/* Self-check of tcgen05 operand layouts written in software: D = A B as in
 * sa_selftest_mma, but both operands are copied into shared memory by the CTA
 * (no TMA), each in its own swizzle: a_sw / b_sw = 128 or 64 (bytes per row of
 * an atom; atoms of 64 or 32 bf16 along the contiguous dimension, which must
 * hold whole atoms).  M in {64, 128}; N, K multiples of 16 up to 256. */
sa_status sa_selftest_mma2(int32_t M, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn, int32_t a_sw,
                           int32_t b_sw, int32_t d_lane, const void* A, const void* B, float* D, int32_t* status,
                           void* stream);

/* Self-check of the TMA row gather the token-level kernels use: n rows (n a
 * multiple of 4, <= 32) of src, a bf16 [rows][cols] matrix (cols a multiple of
 * 64, <= 576), named by row_idx (device int32 [n], each in [0, rows)), are
 * loaded by tile::gather4 copies into 128-byte-swizzled shared memory and
 * written back un-swizzled to out, bf16 [n][cols] (device).  *status (device
 * int32) gets the timeout bit if the wait gives up.  Asynchronous. */
sa_status sa_selftest_gather4(const void* src, int32_t rows, int32_t cols, const int32_t* row_idx, int32_t n,
                              void* out, int32_t* status, void* stream);

/* Self-check of the bounded waits every kernel uses: one CTA waits on an
 * mbarrier that nothing arrives on.  The wait gives up after its poll limit,
 * the kernel ORs the timeout bit (2) into *status (device int32) and returns
 * normally, so the context stays usable; *waited (device int32) gets 1 if the
 * wait (wrongly) completed, else 0.  Asynchronous; takes as long as the limit. */
sa_status sa_selftest_wait_timeout(int32_t* status, int32_t* waited, void* stream);

/* Which kernels sa_fwd and sa_bwd would run for `args` (validated as by
 * *_get_workspace_size).  Either output pointer may be NULL.  Host only. */
sa_status sa_plan(const sa_args* args, int32_t* fwd_kernel, int32_t* bwd_kernel);

/* Read back the status word of a forward or backward workspace (device
 * pointer `ws`, the one the last call on `stream` used): synchronises
 * `stream`, then returns SA_ERR_TIMEOUT if a bounded wait gave up, else
 * SA_ERR_INDEX if an index past its sequence was met, else SA_ERR_CUDA if a
 * kernel could not run, else SA_OK.  The word is left as it is. */
sa_status sa_read_status(const void* ws, size_t ws_bytes, void* stream);

/* The same for the scratch array behind sa_bwd_no_alloc on the current
 * device (after its last call on `stream`). */
sa_status sa_bwd_no_alloc_read_status(void* stream);

/* Block-level index sets exactly as the block kernels build them, for
 * bit-exact checks (64-row blocks, separate K / V).  Each record is four int32
 * {unit = token * Hkv + kv-head, block x, lo, hi}: block x contributes rows
 * [64x + lo, 64x + hi] (sequence-local) to the unit's visible set.
 *   SA_INDEX_VIEW_QUERY_BLOCKS: one record per usable slot of every unit, from
 *     the slot rule and in-block row range of the query-stationary block
 *     kernels (requires SA_KERNEL_FWD_BLOCK for `args`; `ws` unused).
 *   SA_INDEX_VIEW_KEY_LISTS: builds the key-stationary backward's inverse index
 *     into `ws` (a backward workspace of sa_bwd_get_workspace_size bytes) the
 *     way sa_bwd does, then walks every work item as the backward kernel does
 *     and emits one record per (item, token) with the block's row range for
 *     that token (requires a key-stationary backward for `args`).
 * records: device int32 [max_records][4]; *n_records (device int32) receives
 * the number of records produced (may exceed max_records; only max_records
 * are written).  Records come in no particular order.  Asynchronous. */
sa_status sa_debug_block_index(const sa_args* args, int32_t view, void* ws, size_t ws_bytes, int32_t* records,
                               int64_t max_records, int32_t* n_records, void* stream);

/* Human-readable name of a status code (static string). */
const char* sa_status_string(int32_t status);

/* SA_ABI_VERSION of the built library. */
int32_t sa_abi_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SPARSE_ATTN_H_ */
