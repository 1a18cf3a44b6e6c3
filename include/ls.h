/*
 * ls.h -- C ABI of the sparse-attention decode library (sm_100a, NVIDIA B200).
 *
 * One decode step of a DSA-style sparse-attention layer, split into the calls a
 * serving loop makes:
 *
 *   ls_index_score        indexer score of every cached token          (a1)
 *   ls_topk_select        per-request top-k of those scores            (a2)
 *   ls_block_bound_prune  coarse-to-fine indexer: block bounds, prune,  (a3)
 *                         exact re-score of survivors, top-k
 *   ls_hotbuf_resolve     hit/miss of the selection against the HBM    (a4)
 *                         hot buffer, miss compaction, slot replacement
 *   ls_gather_misses      copy missed KV rows from pinned host memory  (a5)
 *   ls_sparse_attn_decode attention over the selected rows only        (a6)
 *   ls_decode_step        a1 (or a3) -> a2 -> [a4 -> a5] -> a6         (a7)
 *
 * Sources.  "LeanSparse: Memory-Efficient Serving for Native Sparse-Attention LLMs"
 * (abstract): sparse attention limits the history each query reads; indexer keys
 * and KV are separate caches reused across steps; coarse-to-fine indexing searches
 * compact representations and retrieves original indexer keys only to refine
 * candidates.  "XM-Sparse: Pushing the Throughput Frontier of Sparse Attention with
 * Netpreme X-Mem" (section on the hot buffer): HBM keeps a per-request hot KV buffer
 * (4,096 tokens) and the indexer-key cache; after each step's selection (2,048 KV)
 * only selected-but-missed KV is fetched from the full history; (section on the KV
 * lifecycle) decode fetches only selected-but-missed KV.  The DSA abstract on the
 * "Related papers: SparseServe" page: attention is restricted to a top-k subset of
 * the cached entries.  The pages print no formulas; the definitions each call
 * implements are stated at the call.
 *
 * Conventions for every call.
 *   - All arrays are caller-owned.  Pointers are CUDA device pointers unless a
 *     field says otherwise.  The library never allocates memory, never frees it,
 *     and never synchronises the stream inside a compute call.
 *   - Calls are asynchronous: they validate their arguments on the host, enqueue
 *     kernels on `stream` and return.  LS_OK means "enqueued".
 *   - Argument errors are reported before anything is launched
 *     (LS_ERR_INVALID_ARG / LS_ERR_UNSUPPORTED); a launch failure gives LS_ERR_CUDA.
 *     ls_get_error_string() then describes the last error of the calling thread.
 *   - Values that only the device knows (lengths, counts, page ids) are checked in
 *     the kernels: an out-of-range value is skipped, never dereferenced, and a bit
 *     is set in the device status word, which ls_check_device_status() reads.
 *   - Integers are int32 unless named int64; "bf16" and "e4m3" arrays hold the raw
 *     bit patterns (uint16 / uint8).  Row-major layouts throughout.
 *   - Pages hold 64 tokens; coarse-to-fine blocks are those same 64-token pages.
 */
#ifndef LS_H_
#define LS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object types as cudaStream_t / cudaEvent_t (and CUstream / CUevent). */
typedef struct CUstream_st* ls_stream_t;
typedef struct CUevent_st* ls_event_t;

typedef enum ls_status {
  LS_OK = 0,
  LS_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, workspace too small */
  LS_ERR_UNSUPPORTED = 2,   /* dtype / shape combination that is not built */
  LS_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  LS_ERR_DEVICE_STATUS = 4  /* a kernel flagged a problem (see ls_check_device_status) */
} ls_status;

typedef enum ls_dtype {
  LS_F32 = 0,
  LS_BF16 = 1,
  LS_E4M3 = 2               /* OCP FP8 E4M3 (bias 7, max 448, no inf) */
} ls_dtype;

/* Device status bits (ls_check_device_status). */
#define LS_DEV_BOUNDS   0x1u  /* an index or length was out of range and was skipped */
#define LS_DEV_TIMEOUT  0x2u  /* a bounded wait inside a kernel gave up */
#define LS_DEV_CAPACITY 0x4u  /* more misses than unpinned hot-buffer slots */

#define LS_PAGE 64            /* tokens per page and per coarse-to-fine block */

/* ------------------------------------------------------------------------------
 * a1. Indexer score.
 *
 *   score[b][s] = key_scale[s] * sum_h (w[b][h] * q_scale[b][h]) * ReLU(q8[b][h] . k8[s])
 *
 * for every cached position s < lens[b] of request b.  Because the scales are
 * positive this equals sum_h w_h * ReLU(q_h . k_s) on the dequantised operands
 * q_h = q_scale_h * e4m3(q8_h), k_s = key_scale_s * e4m3(k8_s) -- the DSA
 * lightning-indexer form; the pages name the indexer keys and scores (LeanSparse,
 * abstract) but print no formula.  Position s of request b lives in physical page
 * page_table[b][s / 64] at row s % 64 of key_pool.
 *
 * Built combinations:
 *   key_dtype LS_E4M3: heads == 64, dim == 128, w_dtype LS_BF16 or LS_F32; q is
 *     e4m3 [B,64,128] with q_scale [B,64]; key_pool e4m3 [num_pages,64,128] with
 *     key_scale [num_pages,64].  tcgen05 fp8 MMA path.
 *   key_dtype LS_F32: 1 <= heads <= 64, 1 <= dim <= 128, dim % 4 == 0; q, w,
 *     key_pool f32; q_scale and key_scale must be NULL.  CUDA-core path.
 * scores[b][s] is written for s < lens[b] only; other entries are left untouched.
 * key_pool and the q rows must be 16-byte aligned.
 * --------------------------------------------------------------------------- */
typedef struct ls_index_score_args {
  int32_t batch;              /* B >= 1 */
  int32_t heads;              /* indexer heads H */
  int32_t dim;                /* indexer head dim D */
  int32_t max_pages;          /* row stride of page_table */
  int32_t max_len;            /* row stride of scores; lens[b] <= min(max_len, 64*max_pages) */
  int32_t key_dtype;          /* ls_dtype: LS_E4M3 or LS_F32 */
  int32_t w_dtype;            /* ls_dtype: LS_BF16 or LS_F32 */
  int32_t variant;            /* 0: fastest built kernel; 1: CUDA-core kernel (any key_dtype) */
  int64_t num_pages;          /* pages in key_pool (page ids must be < num_pages) */
  const void* q;              /* [B,H,D] */
  const float* q_scale;       /* [B,H] (e4m3 only) */
  const void* w;              /* [B,H] head weights */
  const void* key_pool;       /* [num_pages,64,D] */
  const float* key_scale;     /* [num_pages,64] (e4m3 only) */
  const int32_t* page_table;  /* [B,max_pages] */
  const int32_t* lens;        /* [B] */
  float* scores;              /* [B,max_len] out */
} ls_index_score_args;

ls_status ls_index_score(const ls_index_score_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a2. Top-k selection.
 *
 * For each request, the k positions with the largest score (ties: lower position
 * first), written to idx[b][0..k) in ascending position order.  If lens[b] < k the
 * first lens[b] entries are 0..lens[b]-1 and the rest are -1.  sel_score (optional)
 * receives the score of each selected position (0 for padding).  Comparison is on
 * IEEE order with -0 == +0; NaN scores are not supported.  The DSA top-k subset
 * ("Related papers: SparseServe" page, DSA abstract); 2,048 per step in
 * XM-Sparse's hot-buffer section.
 * Limits: 1 <= k <= 4096; scores rows 16-byte aligned (max_len % 4 == 0).
 * --------------------------------------------------------------------------- */
typedef struct ls_topk_args {
  int32_t batch;
  int32_t k;
  int32_t max_len;            /* row stride of scores */
  const float* scores;        /* [B,max_len] */
  const int32_t* lens;        /* [B] */
  int32_t* idx;               /* [B,k] out */
  float* sel_score;           /* [B,k] out, may be NULL */
  const int32_t* pos_offset;  /* optional [B]: added to every emitted position (e.g. the first
                                 position of this GPU's shard of the request); -1 padding stays */
} ls_topk_args;

ls_status ls_topk_select(const ls_topk_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * Block summaries (non-timed helper, run when pages are appended).
 *
 * For each request and 64-token block j: kmax/kmin per dim over the block's valid
 * tokens of k = key_scale * e4m3(k8), stored as e4m3 codes times a float32 block
 * scale bs_j (about amax_j/448, raised by one float32 step when 448*bs_j < amax_j;
 * 1 for an all-zero block), the max rounded up and the min rounded down in exact
 * arithmetic, so the stored box contains every key.  Layout: summaries[b][j] =
 * [kmax codes (D bytes) | kmin codes (D bytes)], block_scale[b][j].
 * LeanSparse (abstract): "coarse-to-fine indexing searches compact representations".
 * Requires key_dtype LS_E4M3, dim 128.
 * --------------------------------------------------------------------------- */
ls_status ls_build_block_summaries(const ls_index_score_args* keys, uint8_t* summaries,
                                   float* block_scale, int32_t max_blocks, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a3. Coarse-to-fine indexer (LeanSparse, abstract: decode can find promising
 * candidates before comparing their original indexer scores; original indexer
 * keys are read only for candidate refinement).  Exact: idx equals what
 * ls_index_score + ls_topk_select return on the same inputs.
 *
 *  1. UB[b][j] = bs_j * sum_h w'_h * ReLU(hi_hj) for w'_h >= 0, w'_h * ReLU(lo_hj)
 *     for w'_h < 0, with w'_h = w_h * q_scale_h and hi/lo = sum_d max/min(q8_hd *
 *     kmax_jd, q8_hd * kmin_jd) -- an upper bound on every score in block j
 *     (for w >= 0: sum_h w_h ReLU(sum_d max(q_hd Kmax_jd, q_hd Kmin_jd))).
 *  2. tau0 = the k-th largest exact score over the ceil(k/64)+1 blocks with the
 *     largest UB (never above the true k-th score).
 *  3. survivors = blocks with UB >= tau0 - eps_j, eps_j = eps_rel * M_j, where
 *     M_j = 448 * bs_j * sum_h |w'_h| * sum_d |e4m3(q8_hd)| bounds |score| in the
 *     block; the margin absorbs float32 rounding so no true top-k block is lost.
 *  4. exact scores of the survivors' tokens, then top-k over them.
 * summaries/block_scale as built by ls_build_block_summaries.  Requires the e4m3
 * indexer (heads 64, dim 128).  idx/sel_score as in ls_topk_select.  survivors
 * receives each request's surviving block ids (ascending), n_survivors the count.
 * Needs a workspace of ls_block_bound_prune_workspace_size() bytes (256-aligned).
 *
 * Host-resident original keys (LeanSparse, abstract: keeping the full indexer keys
 * on the GPU limits decode concurrency): with keys_on_host != 0, index.key_pool and
 * index.key_scale are pinned host memory (cudaHostAlloc / cudaHostRegister, device-
 * accessible); only the summaries stay in HBM.  Steps 2 and 4 first copy the listed
 * blocks' keys and scales (8,448 bytes per block) over the host link into workspace
 * staging of stage_blocks blocks per request, then score them there; survivors beyond
 * stage_blocks take further passes of the same size.  The result is identical to
 * keys in HBM.
 * --------------------------------------------------------------------------- */
typedef struct ls_block_bound_prune_args {
  ls_index_score_args index;  /* a1 inputs; index.scores is ignored */
  int32_t k;
  int32_t max_blocks;         /* row stride of summaries/block_scale/survivors;
                                 >= ceil(lens[b]/64) */
  float eps_rel;              /* <= 0 selects the default 2^-10 */
  const uint8_t* summaries;   /* [B,max_blocks,2*128] e4m3 */
  const float* block_scale;   /* [B,max_blocks] */
  int32_t* idx;               /* [B,k] out */
  float* sel_score;           /* [B,k] out, may be NULL */
  int32_t* survivors;         /* [B,max_blocks] out */
  int32_t* n_survivors;       /* [B] out */
  float* ub;                  /* [B,max_blocks] out, may be NULL */
  int32_t keys_on_host;       /* != 0: index.key_pool / key_scale are pinned host memory */
  int32_t stage_blocks;       /* keys_on_host: staging blocks per request and pass
                                 (0 = 2048; at least ceil(k/64)+1 are used) */
} ls_block_bound_prune_args;

size_t ls_block_bound_prune_workspace_size(const ls_block_bound_prune_args* args);
ls_status ls_block_bound_prune(const ls_block_bound_prune_args* args, void* workspace,
                               size_t workspace_bytes, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a4. Hot-buffer resolve (XM-Sparse, hot-buffer section: a per-request HBM hot
 * buffer; after each step's selection only the selected KV that misses it is
 * fetched).  The pages state no replacement policy; this call implements:
 *   - selection j (sel[b][j] >= 0) hits when slot_of_pos[b][p] >= 0; its slot is
 *     pinned for this step;
 *   - misses are listed in selection order (ascending position) in miss_pos;
 *   - victims are the unpinned slots, empty slots (pos_of_slot == -1) first in slot
 *     order, then occupied slots by (recent_score ascending, slot ascending); the
 *     i-th miss takes the i-th victim (miss_slot[i]); the victim's old position
 *     leaves the buffer (slot_of_pos = -1) and the miss moves in;
 *   - sel_slot[b][j] = the slot that holds selection j after the step (-1 padding);
 *   - recent_score of every selected slot becomes sel_score[b][j].
 * pos_of_slot / slot_of_pos must be mutually inverse on entry and are on exit.
 * k <= n_slots <= 4096 guarantees enough unpinned slots; recent_score must not be
 * NaN.  Only the maps change here: the KV rows move in ls_gather_misses.
 * --------------------------------------------------------------------------- */
typedef struct ls_hotbuf_args {
  int32_t batch;
  int32_t k;
  int32_t n_slots;            /* hot-buffer slots per request (<= 4096) */
  int32_t max_len;            /* row stride of slot_of_pos; positions < max_len */
  const int32_t* sel;         /* [B,k] selected positions, ascending, -1 padded */
  const float* sel_score;     /* [B,k] */
  int32_t* pos_of_slot;       /* [B,n_slots] in/out (-1 = empty) */
  float* recent_score;        /* [B,n_slots] in/out */
  int32_t* slot_of_pos;       /* [B,max_len] in/out (-1 = not resident) */
  int32_t* sel_slot;          /* [B,k] out */
  int32_t* miss_pos;          /* [B,k] out, -1 padded */
  int32_t* miss_slot;         /* [B,k] out, -1 padded */
  int32_t* n_miss;            /* [B] out */
} ls_hotbuf_args;

ls_status ls_hotbuf_resolve(const ls_hotbuf_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a5. Miss gather (XM-Sparse: the full history sits outside HBM; decode fetches
 * only selected-but-missed KV).  For i < n_miss[b]:
 *   hbuf[b][miss_slot[b][i]] = host_kv[page_table[b][p/64]][p%64],  p = miss_pos[b][i]
 * a byte copy of row_bytes per row, read by the SMs straight from pinned host
 * memory in 16-byte vectors.  host_kv is a DEVICE-ACCESSIBLE address of page-locked
 * host memory (the pointer returned by cudaHostAlloc / cudaHostGetDevicePointer;
 * with unified addressing it equals the host pointer).  row_bytes % 16 == 0 and
 * both bases 16-byte aligned.
 * --------------------------------------------------------------------------- */
typedef struct ls_gather_args {
  int32_t batch;
  int32_t k;                  /* row stride of miss_pos / miss_slot */
  int32_t n_slots;
  int32_t max_pages;
  int64_t row_bytes;
  int64_t num_pages;          /* pages in host_kv */
  const void* host_kv;        /* [num_pages,64,row_bytes] pinned host (device-accessible) */
  const int32_t* page_table;  /* [B,max_pages] */
  const int32_t* miss_pos;    /* [B,k] */
  const int32_t* miss_slot;   /* [B,k] */
  const int32_t* n_miss;      /* [B] */
  void* hbuf;                 /* [B,n_slots,row_bytes] */
} ls_gather_args;

ls_status ls_gather_misses(const ls_gather_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a6. Sparse attention decode over the selected rows (LeanSparse, abstract:
 * sparse attention limits the history read by each query).  Per request b and
 * head h, over the selected rows j (sel[b][j] >= 0):
 *   s_j = softmax_scale * q[b][h] . K_j[0:dk];  o[b][h] = sum_j softmax(s)_j V_j[0:dv];
 *   lse[b][h] = log sum_j exp(s_j)   (natural log; -inf and o = 0 if nothing selected)
 * Row address: LS_ROWS_PAGED: row = page_table[b][p/64]*64 + p%64 for position p;
 *              LS_ROWS_SLOTS: row = b*n_slots + slot.
 * K_j = k_rows + row*row_stride, V_j = v_rows + row*row_stride (elements).
 * Built: LS_BF16 MLA-absorbed (heads 128, dk 576, dv 512, one latent KV head, V =
 * the first 512 dims: pass v_rows == k_rows), tcgen05 bf16 MMA path, o bf16;
 *        LS_F32 (heads <= 64, dk, dv <= 128, multiples of 4), CUDA-core path, o f32.
 * Needs a workspace of ls_sparse_attn_workspace_size() bytes (256-aligned).
 * --------------------------------------------------------------------------- */
#define LS_ROWS_PAGED 0
#define LS_ROWS_SLOTS 1

typedef struct ls_sparse_attn_args {
  int32_t batch;
  int32_t heads;
  int32_t dk;
  int32_t dv;
  int32_t k;                  /* row stride of sel */
  int32_t dtype;              /* ls_dtype: LS_BF16 or LS_F32 */
  int32_t variant;            /* 0: fastest built kernel; 1: CUDA-core kernel (any dtype) */
  float softmax_scale;
  int32_t addressing;         /* LS_ROWS_PAGED or LS_ROWS_SLOTS */
  int32_t max_pages;          /* PAGED: row stride of page_table */
  int32_t n_slots;            /* SLOTS: slots per request */
  int64_t row_stride;         /* elements between consecutive rows (>= dk, % 8 == 0) */
  int64_t num_rows;           /* rows addressable from k_rows / v_rows */
  const void* q;              /* [B,heads,dk] */
  const void* k_rows;
  const void* v_rows;
  const int32_t* page_table;  /* PAGED: [B,max_pages] */
  const int32_t* sel;         /* [B,k] positions (PAGED) or slots (SLOTS); -1 skipped */
  void* o;                    /* [B,heads,dv] out: bf16 for bf16 inputs, float32 for f32;
                                 16-byte aligned for the tensor-core kernel.  Device memory,
                                 or pinned host memory the GPU can address (the last kernel
                                 then writes it over the host link) */
  float* lse;                 /* [B,heads] out; device or pinned host memory like o */
  int32_t o_f32;              /* bf16 tensor-core kernel: != 0 writes o as float32, e.g. as a
                                 partial for ls_attn_merge */
} ls_sparse_attn_args;

size_t ls_sparse_attn_workspace_size(const ls_sparse_attn_args* args);
ls_status ls_sparse_attn_decode(const ls_sparse_attn_args* args, void* workspace,
                                size_t workspace_bytes, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * Allocation-free variant of ls_sparse_attn_decode (no counterpart in the paper).
 *
 * For callers that cannot allocate device memory and so cannot hand in a
 * workspace: for example code that runs inside another engine whose memory
 * manager has already reserved the GPU's free HBM for its own pools (a further
 * cudaMalloc there fails or fragments those pools), or a plain C caller that has
 * no device allocator of its own at the point where it decodes.
 *
 * Same arguments, semantics and results as ls_sparse_attn_decode, except that the
 * split-KV partial outputs go to a scratch array built into the library instead of
 * a caller workspace.  The call allocates and frees nothing.
 *   - The scratch holds 20 MiB; every GPU that loads the library holds it until the
 *     process exits.  A configuration whose partials need more returns
 *     LS_ERR_INVALID_ARG with a message (ls_sparse_attn_workspace_size() gives the
 *     need); one that needs none does not touch the scratch.
 *   - The first call in each CUDA context looks up the scratch's device address in
 *     that context (the device's primary context for runtime users, or a context the
 *     caller created and made current); make that first call before any stream capture.
 *     The address is cached under the context's process-unique id, so a context made
 *     after cudaDeviceReset, or a second context on the same device, gets its own
 *     lookup and never a stale address.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents.  Nothing in it has to start at zero: each call writes every partial
 *     before it reads it.  Calls whose kernels overlap on the GPU (for example on two
 *     streams with no ordering between them) race on the array.
 * --------------------------------------------------------------------------- */
ls_status ls_sparse_attn_decode_noalloc(const ls_sparse_attn_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * a7. One decode step: indexer (or coarse-to-fine indexer) -> top-k -> [hot-buffer
 * resolve -> miss gather] -> sparse attention, all on `stream`, with no allocation
 * (the caller provides the workspace) and no host synchronisation.
 *
 * index:   a1 inputs; index.scores may be NULL (then the scores live in workspace).
 * c2f:     use_c2f != 0 selects a3 (summaries required).
 * attn:    a6 inputs; attn.sel / attn.addressing / attn.k are set by the step:
 *          without the hot buffer rows come from attn.k_rows through
 *          index.page_table (paged KV pool in HBM); with it (use_hotbuf != 0) rows
 *          come from the hot buffer `hbuf` through the resolved slots.
 * hot buffer: state arrays as in a4, host history as in a5 (uses index.page_table).
 * idx / sel_score: optional outputs of the selection.
 * events: optional; when non-NULL, events[i] is recorded on `stream` before stage
 *   i (0 indexer, 1 top-k, 2 resolve, 3 gather, 4 attention) and events[5] after
 *   the last stage, so a caller can time each stage.
 * sel_slot / miss_pos / miss_slot: optional outputs of the hot-buffer resolve (as in a4).
 * Selection: with the fp8 tensor-core indexer over whole requests longer than 32,768
 *   tokens (and k <= 6144), the indexer also keeps lists of the scores above a threshold
 *   it derives from the request's own scores, and the top-k selects among them; where a
 *   request's lists are incomplete it selects over all scores.  Either way the selection
 *   equals a2's over the same scores bit for bit.
 * Workspace: needs no initialisation; every count and flag the step keeps there is
 *   reset by the step's own kernels, and whatever an earlier (or failed) call left there
 *   never changes a result (at most it sends a selection to the full path).
 * Streams: the hot-buffer step forks onto two streams of its own and joins back into
 *   `stream`.  Each (host thread, device, caller stream) gets its own pair, created on
 *   first use, so steps issued on independent streams stay independent; steps issued
 *   on one stream reuse it in order.  Device ordinals from 64 up are refused
 *   (LS_ERR_UNSUPPORTED).
 * --------------------------------------------------------------------------- */
typedef struct ls_decode_step_args {
  ls_index_score_args index;
  int32_t k;
  int32_t use_c2f;
  int32_t max_blocks;
  float eps_rel;
  const uint8_t* summaries;
  const float* block_scale;
  int32_t* survivors;         /* c2f: [B,max_blocks] out, may be NULL (workspace) */
  int32_t* n_survivors;       /* c2f: [B] out, may be NULL (workspace) */
  int32_t c2f_keys_on_host;   /* c2f: keys_on_host / stage_blocks of ls_block_bound_prune_args */
  int32_t c2f_stage_blocks;
  ls_sparse_attn_args attn;
  int32_t use_hotbuf;
  int32_t n_slots;
  int32_t* pos_of_slot;
  float* recent_score;
  int32_t* slot_of_pos;       /* [B,index.max_len] */
  const void* host_kv;        /* device-accessible pinned host history [num_pages,64,row_bytes] */
  int64_t host_num_pages;
  void* hbuf;                 /* [B,n_slots,row_bytes] */
  int32_t* n_miss;            /* [B] out, may be NULL (workspace) */
  int32_t* idx;               /* [B,k] out, may be NULL (workspace) */
  float* sel_score;           /* [B,k] out, may be NULL (workspace) */
  ls_event_t* events;         /* NULL or 6 events */
  ls_event_t attn_q_ready;    /* optional: an event the step waits for just before the
                                 attention reads attn.q -- e.g. the end of its host-to-device
                                 copy on another stream, so that copy overlaps the indexer
                                 and top-k; NULL: attn.q is ready when the call is made */
  int32_t* sel_slot;          /* hot buffer: [B,k] out, may be NULL (workspace); as in a4 */
  int32_t* miss_pos;          /* hot buffer: [B,k] out, may be NULL (workspace); as in a4 */
  int32_t* miss_slot;         /* hot buffer: [B,k] out, may be NULL (workspace); as in a4 */
} ls_decode_step_args;

size_t ls_decode_step_workspace_size(const ls_decode_step_args* args);
ls_status ls_decode_step(const ls_decode_step_args* args, void* workspace,
                         size_t workspace_bytes, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * Context-parallel split of one request over G GPUs (no counterpart on the pages'
 * single-GPU path; their 1M-context, batch-4 workload on several GPUs).  GPU g holds
 * the contiguous positions [shard_begin[b], shard_end[b]) of request b, with its own
 * page tables and pools, and per step:
 *   1. ls_index_score + ls_topk_select over its shard, pos_offset = shard_begin, so its
 *      k candidates carry global positions (ascending, -1 padded) and their scores;
 *   2. an all-gather (NCCL, by the caller) of every GPU's candidates into
 *      cand_score / cand_pos [G,B,k], in shard order;
 *   3. ls_cp_merge_topk: the global top-k of the gathered candidates (the same on every
 *      GPU, and the same as one GPU scanning the whole context: scores do not depend on
 *      the shard, ties go to the lower position) and this GPU's part of it as local
 *      positions (-1 elsewhere);
 *   4. ls_sparse_attn_decode over the local part with o_f32 set: a normalised partial
 *      o_g and its lse_g;
 *   5. an all-gather of (o_g, lse_g) and ls_attn_merge:
 *      LSE = ln sum_g exp(lse_g), o = sum_g exp(lse_g - LSE) o_g.
 * --------------------------------------------------------------------------- */
typedef struct ls_cp_merge_args {
  int32_t shards;             /* G */
  int32_t batch;
  int32_t k;
  const float* cand_score;    /* [G,B,k] */
  const int32_t* cand_pos;    /* [G,B,k] global positions, each shard's valid ones first */
  const int32_t* shard_begin; /* [B] this GPU's shard of each request */
  const int32_t* shard_end;   /* [B] */
  int32_t* idx;               /* [B,k] out: global top-k positions, ascending, -1 padded */
  float* sel_score;           /* [B,k] out, may be NULL */
  int32_t* local_sel;         /* [B,k] out, may be NULL: idx - shard_begin inside the shard, else -1 */
} ls_cp_merge_args;

size_t ls_cp_merge_workspace_size(const ls_cp_merge_args* args);
ls_status ls_cp_merge_topk(const ls_cp_merge_args* args, void* workspace, size_t workspace_bytes,
                           ls_stream_t stream);

typedef struct ls_attn_merge_args {
  int32_t parts;              /* G */
  int32_t batch;
  int32_t heads;
  int32_t dv;                 /* multiple of 4 */
  const float* o_parts;       /* [G,B,heads,dv] normalised partial outputs */
  const float* lse_parts;     /* [G,B,heads] their lse (natural log; -inf = empty part) */
  void* o;                    /* [B,heads,dv] out, o_dtype */
  int32_t o_dtype;            /* LS_BF16 or LS_F32 */
  float* lse;                 /* [B,heads] out (-inf and o = 0 when every part is empty) */
} ls_attn_merge_args;

ls_status ls_attn_merge(const ls_attn_merge_args* args, ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * Layer-streaming prefill (LeanSparse, abstract: prefill streams each layer's history
 * through two reusable GPU buffers, so that the full history of every layer never has
 * to sit in HBM at once).
 *
 * For layer l = 0 .. layers-1: the layer's indexer keys and token scales are copied
 * from pinned host memory into one of two staging buffers in the workspace (layer l
 * uses buffer l % 2) on a copy stream owned by the library, while `stream` builds the
 * block summaries of layer l-1 from the other buffer (exactly as
 * ls_build_block_summaries) and, with n_slots > 0, seeds layer l-1's hot buffer.  A
 * buffer is refilled only after the summaries built from it are done.
 *
 * Hot-buffer seed (the pages give no initial contents; this call uses recency): slot
 * s of request b holds position p = lens[b] - n_slots + s when p >= 0, else it is empty
 * (-1); slot_of_pos[b][p] = s for those positions and -1 everywhere else below
 * max_len; recent_score = 0; the seeded rows are copied from host_kv[l] through the
 * page table, as ls_gather_misses does.
 *
 * All pointer arrays ([layers] entries) are read on the host during the call; the
 * pointers in them are device pointers, except host_keys, host_key_scales and host_kv
 * (pinned host memory, device-accessible).  Returns once all work is enqueued; the
 * last operation is on `stream`.  Needs ls_prefill_stream_workspace_size() bytes of
 * workspace (256-byte aligned).
 * --------------------------------------------------------------------------- */
typedef struct ls_prefill_stream_args {
  int32_t layers;
  int32_t batch;
  int32_t max_pages;          /* row stride of page_table */
  int32_t max_len;            /* row stride of slot_of_pos; lens[b] <= min(max_len, 64*max_pages) */
  int32_t max_blocks;         /* row stride of summaries / block_scale; >= ceil(lens[b]/64) */
  int32_t n_slots;            /* hot-buffer slots per request, 0 = no seeding (<= 4096) */
  int64_t num_pages;          /* pages in each layer's pool */
  int64_t row_bytes;          /* seeding: bytes per KV row (multiple of 16) */
  const int32_t* page_table;  /* [B,max_pages], shared by all layers */
  const int32_t* lens;        /* [B] */
  const void* const* host_keys;          /* [layers] -> [num_pages,64,128] e4m3, pinned */
  const float* const* host_key_scales;   /* [layers] -> [num_pages,64] f32, pinned */
  uint8_t* const* summaries;             /* [layers] -> [B,max_blocks,256] out */
  float* const* block_scale;             /* [layers] -> [B,max_blocks] out */
  const void* const* host_kv;            /* [layers] -> [num_pages,64,row_bytes], pinned (seeding) */
  void* const* hbuf;                     /* [layers] -> [B,n_slots,row_bytes] out (seeding) */
  int32_t* const* pos_of_slot;           /* [layers] -> [B,n_slots] out (seeding) */
  int32_t* const* slot_of_pos;           /* [layers] -> [B,max_len] out (seeding) */
  float* const* recent_score;            /* [layers] -> [B,n_slots] out (seeding) */
} ls_prefill_stream_args;

size_t ls_prefill_stream_workspace_size(const ls_prefill_stream_args* args);
ls_status ls_prefill_stream(const ls_prefill_stream_args* args, void* workspace, size_t workspace_bytes,
                            ls_stream_t stream);

/* ------------------------------------------------------------------------------
 * Diagnostics.
 * --------------------------------------------------------------------------- */
/* Every wait inside a kernel (on a barrier or a peer) gives up after a time limit,
 * raises LS_DEV_TIMEOUT in the device status and lets the kernel return; 2 s by
 * default.  ls_set_wait_limit sets it for the current device, in [1 us, 10 s].
 * ls_selftest_bounded_wait launches one wait that nothing completes, so a caller can
 * check that it ends with LS_DEV_TIMEOUT (after the limit) and a usable context. */
ls_status ls_set_wait_limit(uint64_t ns);
ls_status ls_selftest_bounded_wait(ls_stream_t stream);

/* Message of the calling thread's last error (empty string if none). */
const char* ls_get_error_string(void);

/* Synchronises `stream`, returns the device status bits raised since the last
 * check in *flags (may be NULL) and clears them.  LS_OK when no bit was set,
 * LS_ERR_DEVICE_STATUS otherwise.  The status word is per device and shared by all
 * streams. */
ls_status ls_check_device_status(ls_stream_t stream, uint32_t* flags);

/* Library version string. */
const char* ls_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LS_H_ */
