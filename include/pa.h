/*
 * pa.h -- C ABI of the paged-KV attention library (libpa.so), CUDA sm_100a (B200).
 *
 * The library computes attention over a paged KV cache for packed decode and chunked
 * prefill, returning the output and a float32 logsumexp:
 *
 *     out[q, h, :] = softmax_t( scale * Q[q, h, :] . K_s[t, h / G, :] + mask(q, t) ) . V_s[t, h / G, :]
 *     lse[q, h]    = ln sum_t exp( scale * Q[q, h, :] . K_s[t, h / G, :] )   over visible t
 *
 * This is the dense definition of boostr's `standard_attention_fwd` (flash_standard.rs:
 * scores, additive 0/-inf mask, logsumexp cast to F32, softmax times V; query head h reads
 * KV head h / G with G = Hq / Hkv as in `expand_kv`), evaluated over ruDNN's paged layout
 * (paged_attention/mod.rs, `DevicePlan::attention`): packed Q [queries, Hq, D], K cache
 * [pages, page_size, Hkv, D], V cache [pages, page_size, Hkv, Dv], with key t of sequence s
 * in page block_tables[s][t / page_size], slot t % page_size. Neither padded KV gathers nor
 * per-head KV copies are made.
 *
 * Positions and mask. Sequence s has L_s keys (its own new keys included: they are already
 * in the cache) and n_s queries; query j of s sits at absolute position p = L_s - n_s + j
 * (right-aligned: ruDNN "absolute positions ... including prefill chunks", alice-llm
 * "right-aligned causal mask"). Key t is visible to it iff
 *     (!causal || t <= p)  &&  (window == 0 || t + window > p)
 * (boostr `build_attention_mask`: causal masks j > i, a window masks j + window <= i,
 * window 0 is unlimited). A row with no visible key yields out = 0 and lse = -inf.
 *
 * Ownership. Every data pointer is caller-owned device memory on the plan's device,
 * contiguous in the stated layout. The library never synchronises the host with the GPU
 * inside pa_forward / pa_mla_forward and never reads device data back (ruDNN: "no CPU
 * synchronization or host readback").
 *
 * Errors. Every entry point validates all of its arguments before it launches or allocates
 * anything (ruDNN: validate every supplied output before any allocation, clear or launch);
 * on error nothing is launched, a pa_status other than PA_OK is returned, and
 * pa_last_error_message() describes the failure (a thread-local string).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes (ruDNN's PagedAttentionError becomes a code plus a message). */
typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad flag, non-finite or non-positive scale */
    PA_ERR_SHAPE = 2,            /* head counts/dims inconsistent (e.g. Hq % Hkv != 0) */
    PA_ERR_DTYPE = 3,            /* unknown element type */
    PA_ERR_BOUNDS = 4,           /* page id outside the pool, table too narrow, size overflow */
    PA_ERR_ALIAS = 5,            /* out or lse overlaps an input or each other */
    PA_ERR_UNSUPPORTED = 6,      /* valid but not implemented (e.g. head_dim > 1024) */
    PA_ERR_CUDA = 7              /* a CUDA runtime call or kernel launch failed */
} pa_status;

/* Element type of Q, K, V and out (ruDNN accepts F32, F16, BF16). lse is always float32. */
typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1, PA_F16 = 2 } pa_dtype;

/* A cudaStream_t. NULL is the legacy default stream. */
typedef void* pa_stream;

/* Opaque, immutable schedule: per-sequence lengths, query offsets and block tables on the
 * device, plus the plan-owned float32 split workspace. */
typedef struct pa_plan pa_plan;

/*
 * pa_plan_create -- validate a batch schedule and upload it once (ruDNN `DevicePlan::upload`:
 * "creating a new plan is one small upload"; immutable, reusable while the schedule is
 * unchanged).
 *
 *   seq_lens       [num_seqs] host int32: L_s >= 0, keys of sequence s incl. its new ones.
 *   query_offsets  [num_seqs + 1] host int32: prefix sums of n_s, query_offsets[0] == 0,
 *                  0 <= n_s <= L_s. Queries of s are rows query_offsets[s] .. [s+1]-1 of Q.
 *   block_tables   [num_seqs, table_width] host int32, row-major. Entries 0 .. ceil(L_s /
 *                  page_size) - 1 of row s must lie in [0, num_pages); later entries are never
 *                  read and may hold anything (e.g. -1).
 *   page_size      > 0 tokens per page; num_pages >= 0 pages in the pool.
 *   device         CUDA device ordinal, or -1 for a host-only plan: it validates and keeps
 *                  the schedule but owns no device memory, and every forward call on it fails
 *                  with PA_ERR_INVALID_ARGUMENT after validating its own arguments.
 *   upload_stream  stream of the single host-to-device copy (the plan keeps its host copy
 *                  alive, so the caller may free its arrays on return).
 *   out_plan       receives the plan; set to NULL on error.
 *
 * Errors: PA_ERR_INVALID_ARGUMENT (null pointers, negative sizes, n_s > L_s, offsets not
 * starting at 0 or decreasing), PA_ERR_BOUNDS (table too narrow, page id outside the pool),
 * PA_ERR_CUDA (allocation or copy failed).
 */
pa_status pa_plan_create(const int32_t* seq_lens, const int32_t* query_offsets, int32_t num_seqs,
                         const int32_t* block_tables, int32_t table_width, int32_t page_size,
                         int32_t num_pages, int device, pa_stream upload_stream,
                         pa_plan** out_plan);

/* Free the plan's device memory, stream-ordered on the stream of its last call (or its upload
 * stream): work already queued there may still use it, work on other streams must be done.
 * The host does not wait and nothing is queued on the stream but the frees. NULL is a no-op. This is the release of what ruDNN's `DevicePlan`
 * (paged_attention/mod.rs, the struct holding `host: Arc<HostPlan>` and the uploaded
 * `metadata` tensor) owns, which Rust frees when the plan is dropped; the plan-owned split
 * workspace (ruDNN `SplitWorkspace`) and work lists go with it. Returns PA_OK, or PA_ERR_CUDA
 * if the release could not be queued on the stream (the memory is then freed after a stream
 * synchronisation). */
pa_status pa_plan_destroy(pa_plan* plan);

/* Read-only facts about a plan. */
typedef struct pa_plan_info {
    int32_t num_seqs;
    int32_t num_queries;     /* query_offsets[num_seqs] */
    int32_t table_width;
    int32_t page_size;
    int32_t num_pages;
    int32_t device;          /* -1 for a host-only plan */
    int32_t last_launches;   /* kernels the last successful forward call launched */
    int64_t workspace_bytes; /* current size of the plan-owned split workspace */
    int64_t uploaded_bytes;  /* host-to-device bytes the plan has copied (schedule, work lists) */
    int32_t last_kernels;    /* PA_KERNEL_* bits: which kernels the last successful call launched */
} pa_plan_info;

/* Bits of pa_plan_info.last_kernels (which code path served the last call). */
#define PA_KERNEL_DECODE_TC 1u      /* split-KV decode on the tensor cores (mma.sync) */
#define PA_KERNEL_PREFILL_TC 2u     /* chunked prefill on tcgen05 / TMEM / TMA */
#define PA_KERNEL_MLA_TC 4u         /* MLA decode on tcgen05 / TMEM / TMA */
#define PA_KERNEL_SIMT 8u           /* the CUDA-core kernel (fp32, other shapes, PA_PATH_SIMT) */
#define PA_KERNEL_MERGE 16u         /* the split-part merge kernel (CUDA-core, MLA and sparse parts) */
#define PA_KERNEL_SPARSE 32u        /* sparse selection kernels (check, proxy scores, top-K) */
#define PA_KERNEL_APPEND 64u        /* paged append */
#define PA_KERNEL_BACKWARD_TC 128u  /* tensor-core GQA backward */
#define PA_KERNEL_BACKWARD_SIMT 256u /* CUDA-core GQA or MLA backward */
pa_status pa_plan_get_info(const pa_plan* plan, pa_plan_info* info);

/* Path selection (testing and tuning). */
typedef enum pa_path {
    PA_PATH_AUTO = 0, /* tensor-core kernels where the shape allows, CUDA-core kernel elsewhere */
    PA_PATH_SIMT = 1  /* the CUDA-core kernel for every row (any dtype and head size) */
} pa_path;

typedef struct pa_forward_options {
    int32_t kv_chunk; /* keys per split-KV part on the decode paths: 0 = automatic,
                         -1 = never split, > 0 = that many keys per part */
    int32_t path;     /* a pa_path */
    void** trace_events; /* NULL, or three cudaEvent_t recorded on the call's stream: before
                            the attention kernels, between them and the merge kernel, and
                            after the merge kernel (kernel timing without a profiler) */
} pa_forward_options;

/*
 * pa_forward -- paged GQA/MHA attention for every query row of the plan, on `stream`.
 *
 *   q          [N_q, num_q_heads, head_dim]             dtype, N_q = plan's num_queries
 *   k_cache    [num_pages, page_size, num_kv_heads, head_dim]    dtype
 *   v_cache    [num_pages, page_size, num_kv_heads, v_head_dim]  dtype
 *   scale      finite, > 0 (the caller's choice, e.g. 1/sqrt(head_dim))
 *   causal     0 or 1; window >= 0 (0 = no window)
 *   out        [N_q, num_q_heads, v_head_dim] dtype (written; must not overlap any input)
 *   lse        [N_q, num_q_heads] float32 (written; natural log; must not overlap anything)
 *
 * Shapes: num_kv_heads >= 1, num_q_heads % num_kv_heads == 0, 1 <= head_dim, v_head_dim
 * <= 1024 (ruDNN's limit). N_q == 0 returns PA_OK without launching anything.
 * Long contexts are split over several CTAs whose float32 partial results (o_i, lse_i) go to
 * the plan-owned workspace and are merged (ruDNN "split the visible history over multiple planes
 * and merge FP32 statistics"): on the tensor-core decode path by the CTA that completes a row
 * last (plan-owned arrival counters, zero between calls), elsewhere by a second kernel; either
 * way the parts are summed in a fixed order. The workspace grows on demand
 * with stream-ordered allocation on `stream`; calls on one plan must therefore be ordered
 * (one stream, or explicit events). The first call with a new head configuration builds and
 * uploads that configuration's work list once (also available as pa_plan_prepare); make it
 * before capturing the stream into a CUDA graph. A batch with both decode rows and prefill chunks
 * runs its decode kernel on a stream of the library forked from `stream` and joined back into it
 * through events, so the call stays ordered on `stream` (and capturable with it).
 * Inputs must be finite; non-finite values propagate (ruDNN contract).
 */
pa_status pa_forward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                     pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads,
                     int32_t head_dim, int32_t v_head_dim, float scale, int causal,
                     int32_t window, void* out, float* lse, pa_stream stream);

/* pa_forward with options (NULL = defaults). */
pa_status pa_forward_ex(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                        pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads,
                        int32_t head_dim, int32_t v_head_dim, float scale, int causal,
                        int32_t window, void* out, float* lse, pa_stream stream,
                        const pa_forward_options* opts);

/*
 * pa_mla_forward -- MLA absorbed-latent attention (ruDNN `DevicePlan::mla`).
 *
 *   q_latent      [N_q, num_heads, latent_dim]   absorbed queries
 *   q_rope        [N_q, num_heads, rope_dim]     position queries
 *   latent_cache  [num_pages, page_size, 1, latent_dim]  one shared latent head
 *   rope_cache    [num_pages, page_size, 1, rope_dim]
 *   out           [N_q, num_heads, latent_dim]   compressed context (the latent is both key
 *                 and value; the caller applies the value/output projection afterwards)
 *   lse           [N_q, num_heads] float32
 *
 * score(q, h, t) = scale * (q_latent[q,h,:] . latent[t,:] + q_rope[q,h,:] . rope[t,:]);
 * `scale` comes from the original model's QK dimensions, not the latent rank (ruDNN).
 * Shapes: 1 <= latent_dim <= 1024, 1 <= rope_dim <= 256 (ruDNN's positional limit).
 * Same masking, ownership, workspace and error rules as pa_forward.
 */
pa_status pa_mla_forward(pa_plan* plan, const void* q_latent, const void* q_rope,
                         const void* latent_cache, const void* rope_cache, pa_dtype dtype,
                         int32_t num_heads, int32_t latent_dim, int32_t rope_dim, float scale,
                         int causal, int32_t window, void* out, float* lse, pa_stream stream);

pa_status pa_mla_forward_ex(pa_plan* plan, const void* q_latent, const void* q_rope,
                            const void* latent_cache, const void* rope_cache, pa_dtype dtype,
                            int32_t num_heads, int32_t latent_dim, int32_t rope_dim, float scale,
                            int causal, int32_t window, void* out, float* lse, pa_stream stream,
                            const pa_forward_options* opts);

/*
 * pa_append -- write each query row's new key and value into its cache slot (ruDNN
 * `DevicePlan::append`; the step that precedes attention). Query j of sequence s sits at
 * absolute position p = L_s - n_s + j, so its rows go to page block_tables[s][p / page_size],
 * slot p % page_size:
 *   k_cache[page, slot, h, :] = new_k[q, h, :]   and   v_cache[page, slot, h, :] = new_v[q, h, :]
 *
 *   new_k   [N_q, num_kv_heads, head_dim]   dtype (read)
 *   new_v   [N_q, num_kv_heads, v_head_dim] dtype (read)
 *   k_cache [num_pages, page_size, num_kv_heads, head_dim]   (written in place)
 *   v_cache [num_pages, page_size, num_kv_heads, v_head_dim] (written in place)
 * MLA: pass the new latent rows as new_k with the latent cache, and the new rope rows as new_v
 * with the rope cache (num_kv_heads = 1).
 *
 * Rows must be multiples of 16 bytes (PA_ERR_UNSUPPORTED otherwise). The caches must not
 * overlap each other or the new rows (PA_ERR_ALIAS), and no two query rows of the plan may map
 * to one slot (PA_ERR_ALIAS; checked once per plan on the host). The caller owns the caches:
 * this call does not copy shared pages (ruDNN's copy-on-write decision belongs to the caller's
 * page allocator here). Stream-ordered, no host synchronisation.
 */
pa_status pa_append(pa_plan* plan, const void* new_k, const void* new_v, void* k_cache, void* v_cache,
                    pa_dtype dtype, int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim,
                    pa_stream stream);

/*
 * pa_backward -- gradients of paged GQA attention (boostr `standard_attention_bwd`; ruDNN
 * `attention_backward`: weights recomputed from Q and K, not saved). For the upstream gradient
 * d_out of out = softmax(scale Q K^T + mask) V:
 *     dV_t += P_t dO,  dP_t = dO . V_t,  D = dO . out,  dS_t = P_t (dP_t - D),
 *     dQ = scale sum_t dS_t K_t,  dK_t += scale dS_t Q
 * with P recomputed from the forward's lse. Query head h reads KV head h / G, so the G heads of a
 * group (and every query, and every sequence sharing a page) add into the same cache slot.
 *
 *   q, k_cache, v_cache  the forward's inputs (dtype, same layouts as pa_forward)
 *   out, lse             the forward's outputs
 *   d_out                [N_q, Hq, Dv] dtype
 *   d_q                  [N_q, Hq, D] float32, written
 *   d_k_cache            [pages, page_size, Hkv, D] float32, ADDED INTO (zero it first)
 *   d_v_cache            [pages, page_size, Hkv, Dv] float32, ADDED INTO (zero it first)
 * bf16 / fp16 with head_dim == v_head_dim in {64, 128}, G = num_q_heads / num_kv_heads dividing
 * 128, a page size that is a multiple of 16 and divides 128 or is a multiple of 128, fewer than 2^31
 * cache rows and 16-byte aligned q, k_cache, v_cache, d_out, d_k_cache and d_v_cache run on the
 * tensor cores (tcgen05, every operand moved by TMA, K / V one page box at a time): dK/dV key-major
 * (a CTA per 128 keys and KV head, its finished rows added by TMA reduce-adds), dQ query-major (a CTA
 * per 128 rows = 128 / G queries x G heads and KV head, on a second stream of the library that
 * forks from and joins back into `stream`); P and dS are rounded to the input type before the
 * gradient products. Every key's dK/dV row is summed by one CTA and added once; where a page is referenced
 * more than once in the plan (sequences sharing a prefix, a page listed twice), the rows of every key
 * tile that touches it are summed per cache slot in (sequence, key) order by an ordered pass (ruDNN's
 * atomic-free "ordered" history pass), so the result repeats bit for bit in every case (three
 * launches, four with shared pages; the plan keeps the float32 scratch of those tiles). Other shapes
 * and fp32 run a float32 CUDA-core kernel whose dK/dV atomics make the summation order vary between
 * runs (one launch). Validation and errors as pa_forward (gradient outputs must not overlap each
 * other or any input).
 */
pa_status pa_backward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                      const void* out, const float* lse, const void* d_out, pa_dtype dtype,
                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                      int32_t v_head_dim, float scale, int causal, int32_t window, float* d_q,
                      float* d_k_cache, float* d_v_cache, pa_stream stream);

/*
 * pa_mla_backward -- gradients of MLA absorbed-latent attention (the backward the pages list for
 * MLA beside GQA; ruDNN `mla_backward`, recompute-based). MLA is single-head attention with the key
 * [latent | rope] and the value latent, so with P recomputed from the forward's lse:
 *     dP_t = dO . latent_t,  D = dO . out,  dS_t = P_t (dP_t - D)
 *     d_q_latent = scale sum_t dS_t latent_t,    d_q_rope = scale sum_t dS_t rope_t
 *     d_latent_t += scale dS_t q_latent + P_t dO  (the latent is both key and value)
 *     d_rope_t   += scale dS_t q_rope
 * summed over every query head and query that sees key t (and every sequence sharing its page).
 *
 *   q_latent, q_rope, latent_cache, rope_cache   the forward's inputs (dtype; pa_mla_forward layouts)
 *   out, lse                                     the forward's outputs
 *   d_out            [N_q, num_heads, latent_dim] dtype
 *   d_q_latent       [N_q, num_heads, latent_dim] float32, written
 *   d_q_rope         [N_q, num_heads, rope_dim]   float32, written
 *   d_latent_cache   [num_pages, page_size, 1, latent_dim] float32, ADDED INTO (zero it first)
 *   d_rope_cache     [num_pages, page_size, 1, rope_dim]   float32, ADDED INTO (zero it first)
 * bf16 / fp16 with latent_dim 512 and rope_dim 64, every sequence's rows (its queries x num_heads)
 * at most 128, a page size that is a multiple of 16 and divides 128 or is a multiple of 128, fewer
 * than 2^31 cache rows, and no page used by two keys of the plan run on the tensor cores (tcgen05,
 * every operand moved by TMA): a Drow kernel, a key-major kernel (a CTA pair per 128 keys, each
 * owning half of the latent's columns and adding its finished rows once by TMA reduce-adds: the
 * result repeats bit for bit), and a dQ kernel (a CTA per sequence and 64-column chunk of
 * [latent | rope]); P and scale * dS are rounded to the input type before the gradient products.
 * Other shapes, fp32 and plans that share pages run a warp per (query, head) row on the CUDA cores,
 * float32 throughout, with float32 atomics into the cache gradients, so their summation order varies
 * between runs. Shapes as pa_mla_forward; validation and errors as pa_backward (gradient outputs
 * must not overlap each other or any input).
 */
pa_status pa_mla_backward(pa_plan* plan, const void* q_latent, const void* q_rope,
                          const void* latent_cache, const void* rope_cache, const void* out,
                          const float* lse, const void* d_out, pa_dtype dtype, int32_t num_heads,
                          int32_t latent_dim, int32_t rope_dim, float scale, int causal,
                          int32_t window, float* d_q_latent, float* d_q_rope, float* d_latent_cache,
                          float* d_rope_cache, pa_stream stream);

/*
 * pa_forward_static_workspace -- pa_forward's split-KV decode without any memory allocation.
 * The pages describe no such call: it exists for callers that cannot allocate device memory
 * while they run attention (a serving loop that must not stall on the allocator mid-step, a
 * process under a fixed pre-reserved memory budget, a host runtime that forbids cudaMalloc in
 * plugins). pa_forward may allocate: its split workspace grows on demand and the first call with
 * a new head configuration uploads a work list into new memory. This call keeps both in one
 * fixed array of PA_STATIC_WORKSPACE_BYTES in device global memory, defined inside the library;
 * every GPU that loads the library holds that array until the process exits. The caller still
 * provides the plan, the inputs and the outputs, exactly as for pa_forward.
 *
 * Scope: bf16 or fp16, head_dim == v_head_dim in {64, 128}, and every sequence with at most 16
 * query rows per KV head (queries x Hq/Hkv): the tensor-core decode kernel's shapes. Other shapes
 * return PA_ERR_UNSUPPORTED. kv_chunk is pa_forward_options.kv_chunk (0 automatic, -1 never
 * split, > 0 keys per part). A batch whose work list or float32 split parts do not fit the array
 * returns PA_ERR_BOUNDS before anything is launched (a larger kv_chunk, or -1, needs fewer parts).
 *
 * Limits of the array: at most 32768 work units (one per part of a sequence's keys), at most
 * 16384 query rows whose keys are split, and float32 parts of at most the array's size minus
 * 1.25 MiB of unit lists; beyond any of them the call returns PA_ERR_BOUNDS and launches
 * nothing. A sequence whose keys would be cut into more than 1024 parts gets 1024 longer parts
 * (as in pa_forward). The work list is written into the array by a small kernel from the plan's
 * sequence table on the device, so the call makes no host-to-device copy (three launches: the
 * list, the decode, the merge when some row is split).
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, once
 * per device, with that device current). Every call shares the one array and leaves its contents behind; nothing in it
 * needs to start at zero (each call writes its unit lists and every part it later reads).
 * Calls whose GPU work overlaps -- issued on different streams, or from different host threads
 * on different streams -- race on the array: order them on one stream.
 * All other rules (validation before launch, no host synchronisation, errors) are pa_forward's.
 */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)
pa_status pa_forward_static_workspace(pa_plan* plan, const void* q, const void* k_cache,
                                      const void* v_cache, pa_dtype dtype, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim,
                                      float scale, int causal, int32_t window, int32_t kv_chunk,
                                      void* out, float* lse, pa_stream stream);

/*
 * pa_plan_prepare -- build and upload the work list of one head configuration ahead of the
 * first forward call (pa_forward does it implicitly). `mla` selects pa_mla_forward's
 * configuration: num_q_heads is then the head count, head_dim the latent width and v_head_dim
 * the rope width (num_kv_heads is ignored).
 * Uses `stream` for the one upload and the workspace allocation.
 */
pa_status pa_plan_prepare(pa_plan* plan, int mla, pa_dtype dtype, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim,
                          int causal, int32_t window, pa_stream stream,
                          const pa_forward_options* opts);

/*
 * Sparse top-K block attention (alice-llm 2.0.0, sparse_attention/llama3_bridge.rs,
 * `llama3_sparse_attention`): a cheap proxy pass scores fixed-size blocks of keys, each
 * (query, KV head) keeps its top-K blocks, and attention runs over the keys of those blocks only;
 * the per-block partials are merged with the split-KV logsumexp merge (alice-llm `lse_combine`).
 *
 * Blocks. The keys of sequence s are cut into nb_s = ceil(L_s / block_size) blocks of
 * block_size consecutive positions (the last one may be partial; reading of the page's
 * num_pages / (block_size / page_size), which drops a partial last block and would break its
 * "top-K 0 equals dense attention" guarantee). block_size must be a positive multiple of the
 * plan's page_size (the page's BlockPageMismatch rule) and nb_s <= PA_SPARSE_MAX_BLOCKS.
 */
#define PA_SPARSE_MAX_BLOCKS 16384

/*
 * pa_sparse_select -- proxy block scores and top-K block selection, on `stream`.
 *
 * Proxy: for query i of sequence s and KV head h the proxy query is the first query head of
 * the group, q[i, h * G, :] (the page's "cheap proxy = the first Q lane of each KV head"). The
 * score of block b is the largest scaled score scale * q_proxy . k[t, h, :] over the keys t of
 * b that query i can see (causal/window at absolute positions as in pa_forward); a block
 * without a visible key scores -inf. Scores are float32 dot products of the stored values.
 * Selection: k_i = nb_s when topk == 0 or topk >= nb_s (every block: the dense case), else
 * topk; the k_i blocks with the highest scores, equal scores ranking the lower block index
 * first, are written in ascending block order to selection[i, h, 0 .. k_i), and the rest of
 * the row is set to -1.
 *
 *   q, k_cache    as pa_forward (v is not read)
 *   topk          >= 0
 *   selection     [N_q, num_kv_heads, width] int32 device, written; width >= max_s k_s
 *   block_scores  NULL, or [N_q, num_kv_heads, scores_width] float32 device, written with the
 *                 proxy scores (-inf past a sequence's blocks); scores_width >= max_s nb_s
 *
 * Errors: as pa_forward, plus PA_ERR_SHAPE (block_size not a positive multiple of page_size,
 * width or scores_width too small), PA_ERR_UNSUPPORTED (more than PA_SPARSE_MAX_BLOCKS blocks
 * in a sequence), PA_ERR_ALIAS (selection or block_scores overlapping q, k_cache or each other).
 */
pa_status pa_sparse_select(pa_plan* plan, const void* q, const void* k_cache, pa_dtype dtype,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                           int causal, int32_t window, int32_t block_size, int32_t topk,
                           int32_t* selection, int32_t width, float* block_scores,
                           int32_t scores_width, pa_stream stream);

/*
 * pa_sparse_forward -- attention over selected key blocks (alice-llm `kvouter_attention` /
 * `kvouter_forward` + `lse_combine`), on `stream`.
 *
 * Query row (i, h) attends to the keys t of the blocks listed in selection[i, h / G, :] that
 * it can see (causal/window as in pa_forward); out and lse are those of softmax over exactly
 * those keys (a row left with no key gets out = 0, lse = -inf). A selection row holds block
 * indices of its sequence, in any order, and -1 for unused entries; every G query heads of a
 * KV head share its row. The selection is read on the device only: an entry outside
 * [-1, nb_s) or a block listed twice in one row sets the plan's device error word
 * (pa_plan_device_status reports 64) and is skipped; that call's results are then undefined.
 *
 *   q, k_cache, v_cache, dtype, heads, dims, scale, causal, window, out, lse   as pa_forward
 *   block_size   as pa_sparse_select
 *   selection    [N_q, num_kv_heads, width] int32 device (e.g. pa_sparse_select's), width >= 0
 *
 * Errors: as pa_forward, plus PA_ERR_SHAPE for block_size, PA_ERR_UNSUPPORTED for more than
 * PA_SPARSE_MAX_BLOCKS blocks in a sequence, PA_ERR_ALIAS if out or lse overlaps selection.
 */
pa_status pa_sparse_forward(pa_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                            pa_dtype dtype, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t v_head_dim, float scale, int causal,
                            int32_t window, int32_t block_size, const int32_t* selection,
                            int32_t width, void* out, float* lse, pa_stream stream);

/* pa_sparse_forward with options (pa_forward_options: key-part length of the split, counted in
 * keys of the concatenated selected blocks and rounded up to a multiple of 16; path; trace events:
 * the first after the selection check, then around the attention kernels and the merge). */
pa_status pa_sparse_forward_ex(pa_plan* plan, const void* q, const void* k_cache,
                               const void* v_cache, pa_dtype dtype, int32_t num_q_heads,
                               int32_t num_kv_heads, int32_t head_dim, int32_t v_head_dim,
                               float scale, int causal, int32_t window, int32_t block_size,
                               const int32_t* selection, int32_t width, void* out, float* lse,
                               pa_stream stream, const pa_forward_options* opts);

/*
 * pa_plan_device_status -- diagnostic read of the plan's device error word (synchronous copy:
 * not for the hot path). 0 means no kernel reported a failure; a non-zero code means a kernel
 * gave up a bounded wait in its pipeline (the results of that call are undefined).
 */
pa_status pa_plan_device_status(const pa_plan* plan, int32_t* code);

/* Human-readable name of a status code (static string, never NULL; "PA_ERR_UNKNOWN" for a
 * value outside the enum). ruDNN (paged_attention/mod.rs) reports every failure as
 * `PagedAttentionError(&'static str)`, whose `Display` prints that static text; in C the kind of
 * failure becomes the pa_status code named here and the text goes to pa_last_error_message. */
const char* pa_status_string(pa_status status);

/* Message of the last failing call on this thread ("" if none or if the last call succeeded):
 * the text ruDNN carries inside `PagedAttentionError` (paged_attention/mod.rs, e.g. "paged
 * tensor exceeds U32 indexing"), here with the offending values filled in. A thread-local
 * buffer owned by the library: valid until this thread's next call into the library; never
 * free it. */
const char* pa_last_error_message(void);

/* Library version, e.g. "0.1.0". */
const char* pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
