/*
 * sparsekv.h -- C ABI of libsparsekv.so: streaming, block-wise decode
 * attention of a few query tokens over a long paged bf16 KV cache, for
 * NVIDIA B200 (sm_100a).
 *
 * What the calls compute (sources are the pages this library implements):
 *
 *  attn_decode      Softmax attention of each query head over a set of cached
 *                   keys, accumulated 64-token block by block in an online
 *                   softmax state (running max m, sum l, output O), the
 *                   tile-streaming form of "ART (Attention Run-time
 *                   Termination)" section 2.1.  Options:
 *                   - a caller-given traversal order ("ART" 2.4, orthogonal
 *                     ordering layer; full traversal is order-invariant);
 *                   - ART run-time termination ("ART" 2.2 dual threshold,
 *                     2.3 patience, 2.4 block 0 always evaluated first);
 *                   - a sink + recent window, the minimal KV of a sparse layer
 *                     under per-layer hard routing ("Flux Attention" section 2,
 *                     "Efficient Deployment"; 64-token sink as in "Pulsar
 *                     Attention" Phase 1);
 *                   - an explicit list of token segments, e.g. the key ranges of
 *                     selected clusters ("Squeezed Attention", Q2 step 3);
 *                   - a key token range [kv_begin, kv_end), one shard of a
 *                     context split across hosts ("Pulsar Attention" Phase 2).
 *  attn_select_centroids
 *                   Query-centroid comparison and top-k cluster choice
 *                   ("Squeezed Attention", Q2 step 2).
 *  attn_merge_lse   Exact merge of per-shard attention partials by their
 *                   log-sum-exp ("Pulsar Attention" Phase 2, online softmax
 *                   merge).
 *  attn_select_centroids_shared
 *                   The same for a batch of requests over one shared fixed
 *                   context ("Squeezed Attention" Q1: the fixed context is
 *                   clustered once and reused across requests).
 *  attn_select_centroids2
 *                   Two-level (hierarchical) centroid selection ("Squeezed
 *                   Attention", Q2 step 4): coarse clusters first, then the
 *                   fine clusters inside the chosen ones.
 *  attn_forecast, attn_prefetch_blocks
 *                   Lookahead selection of the next layer's KV blocks by a
 *                   Forecast projection, and their prefetch from host memory
 *                   into a device cache ("SparDA", technical summary 2).
 *  attn_route_layers
 *                   Per-layer hard routing between full and sparse attention
 *                   ("Flux Attention" section 2, Layer Router: pooling of the
 *                   query tensor's first and last tokens), with caller-given
 *                   router weights.
 *
 * Conventions (all calls):
 *  - The caller owns and allocates every buffer; the library never allocates
 *    or frees memory.  All pointers below are DEVICE pointers unless stated.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Arguments are validated on the host before any launch; a
 *    non-SKV_OK return means nothing was launched (except SKV_ECUDA, which
 *    reports a launch error).
 *  - No C++ exception or process exit crosses this boundary.
 *  - Problems only the device can see (a page index out of range, a sequence
 *    length above max_seq_len, a traversal entry out of range, a bounded wait
 *    that expired) are OR-ed into *status_word as SKV_DEV_* bits, when
 *    status_word is non-NULL; the affected rows are computed as if the bad
 *    entry were absent.  The caller reads the word back after synchronising.
 *  - Supported shapes: head_dim 128, block_size 64, q_heads / kv_heads in
 *    {1, 2, 4, 8}.  q_tokens == 1 is decode (all options below); q_tokens > 1
 *    is a query chunk computed on the tensor cores (tcgen05): natural
 *    traversal or a [kv_begin, kv_end) range starting on a 64-token block,
 *    optional causal mask over the chunk's own keys, optional equal shards;
 *    no ART, order, window or segments.  Other values return SKV_EUNSUPPORTED.
 *  - Alignment: q, out, k_pool and v_pool 16-byte aligned.
 *  - The first call of each kernel shape on a device sets that kernel's
 *    shared-memory (and cluster) attributes and queries whether a cluster
 *    shape fits; make that first call outside CUDA stream capture.  Later
 *    calls, inside a capture or not, only launch.
 */
#ifndef SPARSEKV_H
#define SPARSEKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SKV_API __attribute__((visibility("default")))
#else
#define SKV_API
#endif

typedef struct CUstream_st* skv_stream_t; /* same type as cudaStream_t */

typedef enum {
  SKV_OK = 0,
  SKV_EINVAL = 1,       /* a bad argument (NULL pointer, size, alignment, threshold) */
  SKV_EUNSUPPORTED = 2, /* valid but not implemented (shape, option combination) */
  SKV_ECUDA = 3,        /* a CUDA runtime call failed (launch, attribute) */
  SKV_ETIMEOUT = 4,     /* a bounded wait inside a kernel expired (skv_status_of_word) */
  SKV_EWORKSPACE = 5    /* workspace NULL or smaller than *_workspace_size */
} skv_status;

/* Bits OR-ed into *status_word by the device. */
#define SKV_DEV_TIMEOUT 0x1u     /* a bounded wait inside a kernel expired */
#define SKV_DEV_BAD_PAGE 0x2u    /* block_table entry < 0 or >= num_pages */
#define SKV_DEV_BAD_SEQLEN 0x4u  /* seq_lens[b] < 0 or > max_seq_len */
#define SKV_DEV_BAD_ORDER 0x8u   /* order entry outside [0, ceil(seq_len/64)) */
#define SKV_DEV_BAD_SEGMENT 0x10u /* segment with start > end */

/* ART run-time termination ("ART" 2.2-2.4).  Per query head, after each
 * consumed block t the probe x_t = first 8 dims of the normalised partial
 * output O_t / l_t is formed; for t >= 1
 *     d_scale = | ||x_t|| - ||x_{t-1}|| | / ||x_{t-1}||
 *     d_dir   = 1 - cos(x_t, x_{t-1})
 * and the test passes when d_scale < tau AND d_dir < phi (strict).  The head
 * stops after `patience` consecutive passes; its output is the attention over
 * the blocks consumed so far.  Zero probes: ||x_{t-1}|| = 0 gives d_scale = 0
 * if ||x_t|| = 0 else +inf; a zero vector gives d_dir = 0 if both are zero,
 * else 1.  tau = phi = 0 never stops (full attention).  Block 0 is always
 * consumed first.  Key loads of a KV group stop once all of its query heads
 * have stopped.  The test is decided per chunk of 16 or 32 blocks, and
 * chunks of the group that started before the stop was decided are read and
 * discarded (cut short every 8 blocks); blocks_consumed counts only the
 * blocks each head attended. */
typedef struct {
  int enable;   /* 0 = off */
  float tau;    /* >= 0, scale-change threshold */
  float phi;    /* >= 0, direction-change threshold */
  int patience; /* >= 1 consecutive passing blocks */
} skv_art;

/* Sink + recent window ("Flux Attention" 2, sparse layers keep minimal KV):
 * attend tokens [0, sink_tokens) U [seq_len - recent_tokens, seq_len), the
 * overlap counted once.  {0, 0} = off. */
typedef struct {
  int sink_tokens;
  int recent_tokens;
} skv_window;

typedef struct {
  const void* q;              /* bf16 [batch][q_tokens][q_heads][head_dim] */
  const void* k_pool;         /* bf16 [num_pages][kv_heads][block_size][head_dim] */
  const void* v_pool;         /* bf16, same layout as k_pool */
  const int32_t* block_table; /* [batch][max_blocks]: logical block j of sequence b
                                 lives in page block_table[b*max_blocks + j] */
  const int32_t* seq_lens;    /* [batch] tokens per sequence, 0 <= seq_len <= max_seq_len */
  const int32_t* order;       /* NULL, or [batch][kv_heads][order_len] logical block ids:
                                 the traversal order.  NULL means natural order
                                 0..nb-1, or with ART recency-first nb-1..1 after
                                 block 0.  With ART, block 0 is visited first and
                                 skipped where it appears in `order`.  Entries are
                                 not deduplicated. */
  int order_len;
  const int32_t* seg_start;   /* NULL, or [batch][kv_heads][n_seg] token ranges */
  const int32_t* seg_end;     /*   [seg_start, seg_end) clipped to [0, seq_len) */
  int n_seg;
  int batch, q_tokens, q_heads, kv_heads, head_dim, block_size;
  int max_blocks;   /* row stride of block_table */
  int num_pages;    /* pages in each pool */
  int max_seq_len;  /* host-side upper bound on seq_lens, used for the launch plan */
  int kv_begin, kv_end; /* if kv_end > 0: attend only tokens in [kv_begin, kv_end) */
  float scale;      /* softmax scale, e.g. 1/sqrt(head_dim) */
  skv_art art;
  skv_window window;
  int causal;       /* q_tokens > 1: the chunk's own keys are the last q_tokens tokens of
                       each sequence; query token t sees positions <= seq_len - q_tokens + t */
  int kv_shards;    /* q_tokens > 1: split [kv_begin, kv_end) (or the whole sequence) into
                       this many equal shards and write one partial per shard: out and lse
                       gain a leading [kv_shards] dimension ("Pulsar Attention" Phase 2
                       local attention per host); 0 or 1 = a single result */
  float* out;               /* fp32 [batch][q_tokens][q_heads][head_dim] */
  float* lse;               /* fp32 [batch][q_tokens][q_heads], natural log of sum exp(scale q.k);
                               -inf (with out = 0) when no key is attended */
  int32_t* blocks_consumed; /* NULL or int32 [batch][q_heads]: KV tiles folded per head */
  uint32_t* status_word;    /* NULL or one device uint32, SKV_DEV_* bits OR-ed in */
  void* workspace;          /* device scratch of skv_decode_workspace_size() bytes */
  size_t workspace_bytes;
} skv_decode_args;

/* Bytes of device workspace attn_decode needs for these arguments (split-KV
 * partials); 0 if none.  Depends only on host-side fields. */
SKV_API size_t skv_decode_workspace_size(const skv_decode_args* args);

/* Kernels one attn_decode call launches for these arguments (1: the walk
 * merges its own partials -- a query chunk, or the split schedule that small
 * walks and segment lists take; 2: the walk, then the record merge), not
 * counting the workspace zeroing (a device memset); 0 if the arguments are
 * invalid.  Depends only on host-side fields; for profiling and accounting. */
SKV_API int skv_decode_launches(const skv_decode_args* args);

/* The launch plan attn_decode would follow for these arguments (host-side
 * fields only; nothing is launched).  For profiling, capacity planning and
 * tests. */
typedef enum {
  SKV_SCHED_PERSISTENT = 0, /* persistent CTAs over all tiles, then the record merge */
  SKV_SCHED_CLUSTER = 1,    /* one cluster of `splits` CTAs per KV group, merged in-kernel */
  SKV_SCHED_ART = 2,        /* ART: persistent CTAs over (chunk, group) items, then the merge */
  SKV_SCHED_CHUNK = 3       /* query chunk (q_tokens > 1) on the tensor cores */
} skv_schedule;

typedef struct {
  int schedule;           /* skv_schedule */
  int ctas;               /* CTAs of the main kernel (cluster schedule: before any halving of
                             a cluster size the device cannot hold; query chunks: 0) */
  int splits;             /* cluster schedule: CTAs per cluster (pieces per KV group); else 0 */
  int art_chunk_blocks;   /* ART: blocks per chunk (16 or 32); else 0 */
  int art_chunks;         /* ART: chunks per KV group (the longest walk's); else 0 */
  int launches;           /* kernels per call, as skv_decode_launches */
  size_t workspace_bytes; /* as skv_decode_workspace_size */
} skv_decode_plan;

/* Fill *plan; SKV_EINVAL for a NULL plan, else attn_decode's validation status. */
SKV_API skv_status skv_decode_plan_info(const skv_decode_args* args, skv_decode_plan* plan);

/* Decode attention, see above.  Option combinations: at most one of
 * {order, window, seg_start/seg_end, kv range}; ART only with natural or
 * `order` traversal.
 * Launch shapes (they follow from host-side fields only):
 *  - long walks: persistent CTAs (2 per SM) share all tiles, then a merge
 *    kernel combines the partial records in the workspace;
 *  - small walks (at most 8 tiles per resident CTA) and segment lists: one
 *    thread-block cluster of up to 16 CTAs per KV group, merged inside the
 *    kernel through distributed shared memory (no workspace); a cluster size
 *    the device cannot hold at once is halved;
 *  - ART: persistent CTAs over (chunk, group) items, then the merge kernel;
 *  - query chunks (q_tokens > 1): one tensor-core kernel.
 * skv_decode_launches and skv_decode_workspace_size report the kernels and
 * the scratch a call needs. */
SKV_API skv_status attn_decode(const skv_decode_args* args, skv_stream_t stream);

/* attn_decode without any allocation -- for callers that cannot allocate.
 * The pages have no counterpart of this call; it is a deployment aid.
 *
 * attn_decode needs device scratch (skv_decode_workspace_size bytes) that the
 * caller normally allocates.  Some callers cannot allocate at the point where
 * they decode (an allocator that must not be re-entered, a hook running
 * inside another library, device memory reserved in full up front).  This
 * call computes exactly what attn_decode computes, with the same arguments
 * (args->workspace and args->workspace_bytes are ignored), but takes its
 * scratch from a fixed array of SKV_STATIC_WORKSPACE_BYTES inside the
 * library's device image, which every GPU that loads the library holds until
 * the process exits.  It calls no allocator.
 *  - Arguments needing more scratch than SKV_STATIC_WORKSPACE_BYTES (see
 *    skv_decode_workspace_size) return SKV_EWORKSPACE and launch nothing.
 *  - The first call on each device looks up the array's device address, with
 *    that device current; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents.
 *    Nothing in it needs to start at zero (every byte read is written earlier
 *    in the same call), but calls that can overlap on the GPU (other streams,
 *    other host threads) race on it: serialise them.
 * Errors: as attn_decode, plus SKV_ECUDA if the address lookup fails.
 * What fits in the array (skv_decode_workspace_size on a 148-SM B200): every
 * walk without ART of up to about 5,500 KV groups at 4 query heads per KV
 * head, 2,800 at 8 (the persistent schedule needs about 17 KiB, or 34 KiB,
 * per resident CTA and per KV group; small walks and segment lists need
 * none), and ART at the Llama-3.1-8B shape (32 query / 8 KV heads) for up to
 * 64 sequences of 32K tokens or 16 of 128K (ART needs 36 to 57 MiB of
 * per-CTA scratch plus about 0.6 KiB per (KV group, chunk, query head)).
 * The device address is
 * looked up once per device and kept for the whole process: it assumes the
 * device's primary context is not reset (cudaDeviceReset) in between. */
#define SKV_STATIC_WORKSPACE_BYTES (96u * 1024u * 1024u)
SKV_API skv_status attn_decode_static_ws(const skv_decode_args* args, skv_stream_t stream);

/* Centroid selection ("Squeezed Attention" Q2 step 2) for each KV group
 * (b, kvh): score_c = (sum over the group's q_heads/kv_heads query heads of
 * q_h) . centroid_c, c in [0, n_clusters); keep the `topk` largest, ties to the
 * lower index; write the kept ids in ascending order and their key ranges
 *   seg_start[i] = cluster_off[id_i], seg_end[i] = cluster_off[id_i + 1].
 *  q           bf16 [batch][q_heads][head_dim] (one query token)
 *  centroids   bf16 [batch][kv_heads][n_clusters][head_dim]
 *  cluster_off int32 [batch][kv_heads][n_clusters + 1], cluster c holds the
 *              cache tokens [cluster_off[c], cluster_off[c+1])
 *  sel_ids, seg_start, seg_end  int32 [batch][kv_heads][topk] (outputs)
 * Supported: head_dim 128, 1 <= topk <= n_clusters <= 4096. */
SKV_API skv_status attn_select_centroids(const void* q, const void* centroids, const int32_t* cluster_off,
                                 int batch, int q_heads, int kv_heads, int head_dim,
                                 int n_clusters, int topk, int32_t* sel_ids, int32_t* seg_start,
                                 int32_t* seg_end, skv_stream_t stream);

/* Centroid selection over ONE shared fixed context ("Squeezed Attention" Q1:
 * the fixed part of the prompt is clustered offline once and reused by every
 * request; Q2 step 2 per request).  Every request b of the batch has its own
 * query, all requests share one centroid set and one key layout per KV head:
 *   score_c(b, kvh) = (sum of request b's query heads of KV head kvh) . centroid[kvh][c]
 * and the kept clusters follow the same rule as attn_select_centroids (top
 * `topk`, ties to the lower index, ids ascending, key ranges from
 * cluster_off[kvh]).  Up to 8 requests are served together: each centroid row
 * is read once for all of them.
 *  q           bf16 [batch][q_heads][head_dim] (one query token per request)
 *  centroids   bf16 [kv_heads][n_clusters][head_dim] (shared)
 *  cluster_off int32 [kv_heads][n_clusters + 1] (shared)
 *  sel_ids, seg_start, seg_end  int32 [batch][kv_heads][topk] (outputs)
 * The selected ranges index the shared context: attend them with attn_decode
 * (segments) over a block_table whose rows map every request to the same
 * pages.  Supported: head_dim 128, 1 <= topk <= n_clusters <= 4096. */
SKV_API skv_status attn_select_centroids_shared(const void* q, const void* centroids,
                                        const int32_t* cluster_off, int batch, int q_heads,
                                        int kv_heads, int head_dim, int n_clusters, int topk,
                                        int32_t* sel_ids, int32_t* seg_start, int32_t* seg_end,
                                        skv_stream_t stream);

/* Two-level centroid selection ("Squeezed Attention" Q2 step 4, hierarchical
 * clustering) for each KV group (b, kvh), with the group's query heads summed
 * as in attn_select_centroids:
 *   1. score the n_coarse coarse centroids, keep the k1 best (ties to the
 *      lower id);
 *   2. the candidates are the fine clusters of the kept coarse clusters
 *      (coarse cluster i owns fine clusters coarse_off[i] .. coarse_off[i+1]-1);
 *   3. score only the candidates' fine centroids and keep the
 *      min(k2, #candidates) best (ties to the lower fine id).
 * The kept fine ids are written ascending with their key ranges
 *   seg_start[i] = cluster_off[id_i], seg_end[i] = cluster_off[id_i + 1];
 * unused slots get id -1 and an empty range [0, 0) (which attn_decode's
 * segment traversal attends as nothing).
 *  q           bf16 [batch][q_heads][head_dim] (one query token)
 *  coarse      bf16 [batch][kv_heads][n_coarse][head_dim], 16-byte aligned
 *  coarse_off  int32 [batch][kv_heads][n_coarse + 1], within [0, n_fine]
 *  fine        bf16 [batch][kv_heads][n_fine][head_dim], 16-byte aligned
 *  cluster_off int32 [batch][kv_heads][n_fine + 1]: fine cluster f holds the
 *              cache tokens [cluster_off[f], cluster_off[f+1])
 *  sel_ids, seg_start, seg_end  int32 [batch][kv_heads][k2] (outputs)
 * Supported: head_dim 128, n_coarse <= 1024, n_fine <= 4096; 1 <= k1 <=
 * n_coarse, 1 <= k2 <= n_fine (else SKV_EINVAL).  coarse_off ranges are
 * clamped to [0, n_fine). */
SKV_API skv_status attn_select_centroids2(const void* q, const void* coarse, const int32_t* coarse_off,
                                  const void* fine, const int32_t* cluster_off, int batch,
                                  int q_heads, int kv_heads, int head_dim, int n_coarse,
                                  int n_fine, int k1, int k2, int32_t* sel_ids,
                                  int32_t* seg_start, int32_t* seg_end, skv_stream_t stream);

/* Exact LSE merge ("Pulsar Attention" Phase 2) of n_parts partials of n_rows
 * rows each:
 *   M = max_s lse_s,  w_s = exp(lse_s - M),
 *   out = sum_s w_s o_s / sum_s w_s,  lse = M + log sum_s w_s.
 * A partial with lse = -inf has weight 0; if all are -inf, out = 0 and
 * lse = -inf.
 *  o_parts   fp32 [n_parts][n_rows][head_dim] (each row normalised)
 *  lse_parts fp32 [n_parts][n_rows]
 *  out       fp32 [n_rows][head_dim], lse fp32 [n_rows]
 * head_dim must be a multiple of 4 and <= 512; 16-byte aligned o_parts/out. */
SKV_API skv_status attn_merge_lse(const float* o_parts, const float* lse_parts, int n_parts, int n_rows,
                          int head_dim, float* out, float* lse, skv_stream_t stream);

/* Per-layer hard routing ("Flux Attention" section 2: a Layer Router pools
 * the first and last tokens of the input query tensor and decides, per layer,
 * full attention (FA) or sparse attention (SA); inference uses the hard
 * decision, made once per prefill).  For layer l and sequence b, with
 * F = q_heads * head_dim:
 *   p = mean over t <  n_prefix          of q[l][b][t][:]
 *   s = mean over t >= tokens - n_suffix of q[l][b][t][:]
 *   z = w[l][0:F] . p + w[l][F:2F] . s + bias[l]
 *   route[l][b] = z > 0 ? 1 (FA) : 0 (SA);   logits[l][b] = z
 * The prefix and suffix may overlap.  The router's weights come from the
 * caller (the pages train them; this call only applies them).
 *  q       bf16 [n_layers][batch][tokens][q_heads][head_dim], 16-byte aligned
 *  w       fp32 [n_layers][2 * F], 16-byte aligned
 *  bias    fp32 [n_layers], or NULL for zero
 *  logits  fp32 [n_layers][batch], or NULL
 *  route   uint8 [n_layers][batch]
 * Errors: SKV_EINVAL for a NULL q/w/route, a non-positive size, n_prefix or
 * n_suffix outside [1, tokens], or misalignment; SKV_EUNSUPPORTED if F is not
 * a multiple of 8 or n_layers > 65535; SKV_ECUDA if the launch fails. */
SKV_API skv_status attn_route_layers(const void* q, const float* w, const float* bias, int n_layers,
                             int batch, int tokens, int q_heads, int head_dim, int n_prefix,
                             int n_suffix, float* logits, uint8_t* route, skv_stream_t stream);

/* Lookahead block selection and prefetch from host memory ("SparDA",
 * technical summary section 2: "Trainable Lookahead Sparse Selection" and
 * "Asynchronous Prefetch with Persistent UVA Kernel").  Layer l's Forecast
 * projection F_l (one head per GQA group) predicts the top-k KV blocks that
 * layer l+1 needs; while layer l runs, those blocks are pulled from CPU
 * memory into a small device cache, and layer l+1 attends them there.
 *
 * attn_forecast: f[b][kvh] = bf16( W[kvh]^T x[b][kvh] ) for every request b
 * and KV head kvh: output dim j accumulates w[kvh][i][j] * x[b][kvh][i] in
 * fp32 with fused multiply-adds in order i = 0 .. head_dim-1, then rounds to
 * bf16 (nearest even).  Untrained weights make this a random projection.
 *  x  bf16 [batch][kv_heads][head_dim]   the layer-l activation per GQA group
 *  w  bf16 [kv_heads][head_dim][head_dim] (input dim major)
 *  f  bf16 [batch][kv_heads][head_dim]   (output)
 * The block choice is then attn_select_centroids with q = f (q_heads =
 * kv_heads), the block summaries of layer l+1 as the centroids and the block
 * boundaries (j * 64, clipped to the sequence) as cluster_off.
 * Supported: head_dim 128; batch, kv_heads <= 65535. */
SKV_API skv_status attn_forecast(const void* x, const void* w, int batch, int kv_heads, int head_dim,
                                 void* f, skv_stream_t stream);

/* Device-accessible address of page-locked host memory (allocated with
 * cudaHostAlloc, or registered with cudaHostRegister and mapped); under
 * unified addressing it is the host address itself.  SKV_EINVAL if the memory
 * is not page-locked and mapped.  Not stream-ordered: call it at set-up, not
 * during stream capture. */
SKV_API skv_status skv_host_device_pointer(const void* host, void** dev);

/* attn_prefetch_blocks: copy the chosen blocks from a host KV pool into a
 * device cache.  n_ctas CTAs walk the (b, kvh, i) items; item (b, kvh, i)
 * copies logical block j = block_ids[b][kvh][i] of sequence b (its page
 * block_table[b][j] of the host pools, K and V rows of KV head kvh) into page
 * b * topk + i of the cache pools (slot kvh), read from host memory with
 * 16-byte loads through the pools' device-accessible addresses, and writes
 * the slot's token range in the cache
 *     seg_start[b][kvh][i] = i * 64,  seg_end = i * 64 + (tokens of block j)
 * (an empty range for block_ids = -1 or a block at or past the sequence's
 * end, as an empty cluster contributes no keys).  attn_decode with these segments, the
 * cache pools and a block table with row b = b*topk .. b*topk + topk - 1 then
 * attends exactly the chosen blocks.  Rows of the cache past a block's last
 * token are left untouched.
 *  k_host, v_host  device-accessible addresses (skv_host_device_pointer) of
 *                  page-locked bf16 pools [num_pages][kv_heads][64][head_dim]
 *  block_table     int32 [batch][max_blocks] (device), pages of the host pools
 *  seq_lens        int32 [batch] (device)
 *  block_ids       int32 [batch][kv_heads][topk] (device), e.g. from
 *                  attn_select_centroids
 *  k_cache, v_cache bf16 [batch * topk][kv_heads][64][head_dim] (device)
 *  seg_start, seg_end int32 [batch][kv_heads][topk] (device, outputs)
 *  status_word     NULL or a device uint32: SKV_DEV_BAD_PAGE and _BAD_SEQLEN
 *                  are OR-ed in and the item copies nothing
 * Its CTAs are small (64 threads, no shared memory) so that they fit on an
 * SM beside two CTAs of the decode kernels: launch it on its own stream next
 * to the attention it should overlap.  Alone, about 32 CTAs keep a PCIe link
 * busy; beside an attention kernel each resident CTA also slows that kernel,
 * so the fastest pair uses fewer (about 20 beside a 0.8 ms layer on B200).
 * Supported: head_dim 128; 16-byte aligned pools and caches. */
SKV_API skv_status attn_prefetch_blocks(const void* k_host, const void* v_host,
                                        const int32_t* block_table, const int32_t* seq_lens,
                                        const int32_t* block_ids, int batch, int kv_heads,
                                        int head_dim, int topk, int max_blocks, int num_pages,
                                        int max_seq_len, void* k_cache, void* v_cache,
                                        int32_t* seg_start, int32_t* seg_end,
                                        uint32_t* status_word, int n_ctas, skv_stream_t stream);

/* The status a device status word stands for, once the caller has read it
 * back after synchronising: SKV_ETIMEOUT if SKV_DEV_TIMEOUT is set (a bounded
 * wait expired; the affected outputs are not valid), else SKV_EINVAL if any
 * bad-input bit is set (SKV_DEV_BAD_*; the bad entries were skipped), else
 * SKV_OK.  Host-only; no CUDA call. */
SKV_API skv_status skv_status_of_word(uint32_t status_word);

/* Test hook for failure detection, not for production use.  The NEXT
 * attn_decode call that runs the plain decode kernel (no ART, q_tokens == 1)
 * makes the producer warp of CTA `cta` (linear block index) stop before ring
 * entry `entry` (0-based): that entry and everything after it in the CTA are
 * never issued, so the CTA's consumers wait for it until their bounded wait
 * (1 s) expires, set SKV_DEV_TIMEOUT in *status_word, drain the copies in
 * flight and return; the call's outputs are then not valid.  Nothing faults
 * and nothing hangs.  One-shot (the call that takes it clears it); a CTA or
 * entry the launch does not reach leaves the launch unaffected.  cta < 0
 * clears a pending hook; SKV_EINVAL for cta >= 0 and entry < 0. */
SKV_API skv_status skv_test_withhold_tile(int cta, int entry);

/* Static description of a status code. */
SKV_API const char* skv_strerror(skv_status s);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEKV_H */
