/*
 * mk.h -- C ABI of the persistent decode megakernel for B200 (sm_100a).
 *
 * One Llama-style decoder step (RMSNorm, QKV projection + RoPE, KV-cache append, decode
 * attention, O-projection + residual, SwiGLU MLP, final norm + LM head) is lowered on the
 * host into a task graph of tiles linked by dependency events, and one persistent kernel
 * with one CTA per SM runs the whole step.  The method is the one described in
 * "Compiler des LLM en MegaKernel pour obtenir une inference a faible latence"
 * (fr.news.hada.io summary of the Mirage Persistent Kernel post): Part 1 "Compilateur"
 * (computation graph -> task graph of tasks and events), Part 2 "Runtime" (workers,
 * schedulers, event-driven execution).  The per-op definitions follow the Mirage article
 * (iaiol.com): the attention example O = softmax(Q K) V, "Case 1: Normalization + Linear"
 * and "Case 3: Gated MLP".
 *
 * Conventions for every entry point:
 *   - Plain C types only.  `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Device pointers are raw CUDA device addresses the CALLER owns
 *     (allocated e.g. with torch); the library never frees them.
 *   - Calls that take a stream are asynchronous and stream-ordered.
 *   - Every int-returning function returns MK_OK (0) or a negative MK_ERR_* code and never
 *     aborts or throws.  mk_last_error() then holds a one-line description.
 *   - Device-side timeouts (a dependency wait that ran out) are reported by the next
 *     mk_sync_status() on the stream that ran the step.
 *   - bf16 / fp16 values are passed as uint16_t bit patterns.
 */
#ifndef MK_H
#define MK_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MK_OK 0
#define MK_ERR_INVALID_ARG (-1)    /* a pointer, size or config field is out of range */
#define MK_ERR_CUDA (-2)           /* a CUDA runtime call failed (text in mk_last_error) */
#define MK_ERR_DEVICE_TIMEOUT (-3) /* a device-side dependency wait exceeded its limit */
#define MK_ERR_NOT_RESIDENT (-4)   /* the persistent grid cannot be co-resident on the GPU */
#define MK_ERR_STATE (-5)          /* call out of order (e.g. decode before load) */
#define MK_ERR_UNSUPPORTED (-6)    /* valid config this build has no kernel instantiation for */

/* Model and capacity.  Decoder shape as in the pages' workloads (Llama-3-8B shape for the
 * MPK decode benchmark, "Valeur cle de MPK"; Chameleon-7B / Llama-3-8B shapes in the Mirage
 * article's end-to-end figure).  Requirements checked by mk_build_taskgraph:
 * hidden == n_q_heads * head_dim; n_q_heads % n_kv_heads == 0; head_dim in {64, 128};
 * hidden and ffn multiples of 8; max_batch in [1, MK_MAX_BATCH]; tie_embeddings == 0;
 * qk_norm in {0, 1}. */
typedef struct mk_config {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  float rms_eps, rope_theta;
  int max_batch, max_seq;
  int tie_embeddings; /* must be 0: separate LM-head matrix */
  /* 1: QK-norm (Mirage article, "Case 4.1: Attention with Query-Key Normalization", as in
   * Chameleon): every query head and key head of the QKV projection goes through a LayerNorm
   * over its head_dim values (mean and mean squared deviation, eps = rms_eps) with a gain and
   * a bias per head and element, before RoPE; the cache holds the normalised, rotated keys.
   * 0: none. */
  int qk_norm;
  /* Smallest max_batch served by the tensor-core instantiation (the projections as 128-row
   * tcgen05 tiles over N = 32 columns: 16 sequences' high and low bf16 parts, unused ones
   * zero); smaller batches take the CUDA-core GEMV (width 1, or width 4 for 2..4 sequences).
   * 2..5, or 0 for the default 2: every batched width on the tensor cores (on B200 batch 4
   * runs 20 % faster there than on the width-4 GEMV).  5 keeps batches 2..4 on CUDA cores. */
  int tc_min_batch;
} mk_config;

#define MK_MAX_BATCH 16

/* Host weights: bf16 bit patterns, canonical [out, in] row-major; per-layer arrays hold
 * n_layers pointers.  Read once by mk_load_weights; the caller keeps ownership. */
typedef struct mk_host_weights {
  const uint16_t* embed;      /* [vocab, hidden] */
  const uint16_t* lm_head;    /* [vocab, hidden] */
  const uint16_t* final_norm; /* [hidden] */
  const uint16_t* const* attn_norm; /* [hidden] */
  const uint16_t* const* wq;  /* [n_q_heads*head_dim, hidden] */
  const uint16_t* const* wk;  /* [n_kv_heads*head_dim, hidden] */
  const uint16_t* const* wv;  /* [n_kv_heads*head_dim, hidden] */
  const uint16_t* const* wo;  /* [hidden, n_q_heads*head_dim] */
  const uint16_t* const* mlp_norm; /* [hidden] */
  const uint16_t* const* wg;  /* [ffn, hidden] */
  const uint16_t* const* wu;  /* [ffn, hidden] */
  const uint16_t* const* wd;  /* [hidden, ffn] */
  /* QK-norm gains and biases (required when cfg.qk_norm, ignored otherwise):
   * q_norm_* [n_q_heads*head_dim] (head h at h*head_dim), k_norm_* [n_kv_heads*head_dim]. */
  const uint16_t* const* q_norm_w;
  const uint16_t* const* q_norm_b;
  const uint16_t* const* k_norm_w;
  const uint16_t* const* k_norm_b;
} mk_host_weights;

typedef struct mk_ctx mk_ctx; /* opaque, library-owned host object */

/* Lower one decoder step of `cfg` into the task graph for `device` (Part 1 "Compilateur":
 * every op split into per-SM tile tasks; events with thresholds equal to their producer
 * counts; per-SM queues in a topological order), validate it on the CPU (acyclic, counts
 * consistent, every read ordered after its writes, no queue can deadlock) and size the
 * arenas.  Allocates no device memory.  *out receives the context (NULL on error). */
int mk_build_taskgraph(const mk_config* cfg, int device, mk_ctx** out);

/* Sizes (bytes) of the three device buffers the caller allocates.  The weight arena holds
 * the packed bf16 weights; the workspace holds the task graph, event counters, activations
 * and prefill scratch; the KV cache is bf16 in the layout
 * [layer][K=0|V=1][max_batch][n_kv_heads][max_seq][head_dim].  All need 256-byte alignment. */
size_t mk_weight_arena_bytes(const mk_ctx* ctx);
size_t mk_workspace_bytes(const mk_ctx* ctx);
size_t mk_kv_cache_bytes(const mk_ctx* ctx);

/* Pack the host weights into tile order (QKV rows grouped per KV head with RoPE pairs
 * adjacent; gate/up rows interleaved) and copy them to `weight_arena`; upload the task
 * graph and RoPE table into `workspace` and zero its event counters.  The packing depends
 * on max_batch: row-major for 1 sequence; W_down in K chunks of 4096 columns for 2..4;
 * every projection in 128 x 128 blocks of tensor-core core matrices for 5..16.  Both
 * buffers must stay allocated and unmoved until mk_destroy.  Synchronises `stream` before
 * returning. */
int mk_load_weights(mk_ctx* ctx, const mk_host_weights* w, void* weight_arena, void* workspace, void* stream);

/* Prefill (the hybrid arrangement of "Ada-MK: Adaptive MegaKernel Optimization via
 * Automated DAG-based Search for LLM Inference", section 3: prompt on ordinary kernels,
 * decode on the megakernel).  tokens: device int32 [B][T]; fills positions 0..T-1 of
 * the cache for sequences 0..B-1 and sets their positions to T.  last_logits: device fp32
 * [B][vocab] for the last prompt token, or NULL.  B <= max_batch, T <= max_seq. */
int mk_prefill(mk_ctx* ctx, const int32_t* tokens, int B, int T, void* kv_cache, float* last_logits,
               void* stream);

/* Declare that the caller filled the cache itself: sequence b (b < B) has host_pos[b]
 * valid positions.  Sets the active batch to B.  The cache holds keys as the decoder stores
 * them: rotated by RoPE and, with qk_norm, normalised before that. */
int mk_set_positions(mk_ctx* ctx, const int32_t* host_pos, int B);
/* Current positions of the active batch (host copy kept by the library); returns B. */
int mk_get_positions(const mk_ctx* ctx, int32_t* host_pos, int capacity);

/* One decode step of the active batch: one launch of the persistent megakernel.
 * tokens: device int32 [B], token b goes in at position pos[b]; logits: device fp32
 * [B][vocab]; next_tokens: device int32 [B] (greedy argmax, lowest index on ties) or NULL.
 * Appends K/V at pos[b] and advances every position by one.  The kernel serves up to 1
 * (max_batch 1), 4 (max_batch 2..4, CUDA-core GEMV) or 16 (max_batch 5..16, projections as
 * tcgen05 tensor-core tiles) sequences; sequences past B are masked.  MK_ERR_INVALID_ARG if
 * a sequence is full (pos = max_seq); MK_ERR_UNSUPPORTED if no kernel instantiation exists
 * for the shape. */
int mk_decode_step(mk_ctx* ctx, const int32_t* tokens, void* kv_cache, float* logits, int32_t* next_tokens,
                   void* stream);

/* Several greedy decode steps in ONE launch of the persistent megakernel (the token picked
 * by step s, lowest index on ties, is the input of step s + 1 without leaving the device).
 * tokens: device int32 [B] for the first step; tokens_out: device int32 [n_steps][max_batch]
 * (row s, entries b < B: the token picked by step s; required); logits: device fp32
 * [B][vocab], left holding the
 * last step's.  1 <= n_steps <= MK_MAX_STEPS and pos[b] + n_steps <= max_seq, else
 * MK_ERR_INVALID_ARG.  The result equals n_steps mk_decode_step calls fed with their own
 * picks.  Inside the launch, cache rows written by its earlier steps are read from memory
 * after their producers finished, not streamed ahead. */
#define MK_MAX_STEPS 4096
int mk_decode_steps(mk_ctx* ctx, const int32_t* tokens, int n_steps, void* kv_cache, float* logits,
                    int32_t* tokens_out, void* stream);

/* Synchronise `stream` and report the device status of the steps run on it:
 * MK_OK, or MK_ERR_DEVICE_TIMEOUT (the event counters are then reset so the context
 * stays usable; the cache contents of the failed step are undefined). */
int mk_sync_status(mk_ctx* ctx, void* stream);

/* Limit of every device-side wait, in nanoseconds (default 2e9).  Must be > 0. */
int mk_set_wait_timeout_ns(mk_ctx* ctx, uint64_t ns);

/* Test hook for failure detection: while `on` is nonzero, the next decode steps skip the
 * notify of event `event_id` (as if its producer never finished), so every task waiting
 * on it times out after the wait limit and the step reports MK_ERR_DEVICE_TIMEOUT.
 * Nothing faults or traps. */
int mk_debug_drop_notify(mk_ctx* ctx, int event_id, int on);

/* Calibrated static schedule: re-partition every projection's rows over the SMs in
 * proportion to weights[s] (relative streaming speed of SM s, n = mk_get_graph_info().n_sms;
 * equal weights = equal bytes per SM, the default).  On this GPU some SMs stream measurably
 * slower, and with equal shares every phase waits for them; weights measured from traced
 * steps (see the binding's Megakernel.calibrate) fix the schedule offline, as the fixed
 * schedule found ahead of time in "Ada-MK ..." section 2.  The new graph is validated like
 * the first one; if weights are already loaded it is uploaded at once (after synchronising
 * `stream`) and the event counters restart.  Returns MK_ERR_UNSUPPORTED if the new graph
 * does not fit the workspace reserve (the old graph then stays). */
int mk_set_sm_weights(mk_ctx* ctx, const float* weights, int n, void* stream);

/* The same for one projection only: op_kind 2 (QKV), 4 (O), 5 (gate/up), 6 (down) or 7 (LM
 * head) takes its rows by `weights`, the other projections keep theirs (an SM can be slow in
 * one phase only, e.g. where it also runs attention).  mk_set_sm_weights resets every
 * projection to its weights.  Errors as mk_set_sm_weights; MK_ERR_INVALID_ARG for another
 * op_kind. */
int mk_set_op_sm_weights(mk_ctx* ctx, int op_kind, const float* weights, int n, void* stream);

/* Scheduling variant (MPK's run-time dispatch vs the static schedule of "Ada-MK: Adaptive
 * MegaKernel Optimization via Automated DAG-based Search for LLM Inference", section 2).
 * MK_DISPATCH_STATIC (default): every task has a fixed SM and queue position, chosen at
 * lowering time.  MK_DISPATCH_CLAIM: every projection of every layer becomes a pool of
 * tasks_per_sm * n_sms equal tasks (1..4); each SM's queue holds one entry per pool, where the
 * SM claims tasks from the pool's counter (one atomic add per claim) until it is empty, so
 * faster SMs take more; attention, embedding and LM-head tasks stay static.  The graph is
 * validated with the pools' tasks dealt round-robin.  MK_DISPATCH_CLAIM_PACED: the same, but an
 * SM claims its next task only once its workers finished every task but the last one handed
 * to them (at most one unstarted claimed task per SM).  Only the batch-1 kernel of the Llama-3-8B
 * and tiny shapes has a run-time-claim instantiation: MK_ERR_UNSUPPORTED otherwise.  Rebuilds
 * and re-uploads the graph (synchronises `stream` first if weights are loaded). */
#define MK_DISPATCH_STATIC 0
#define MK_DISPATCH_CLAIM 1
#define MK_DISPATCH_CLAIM_PACED 2
/* Priority dispatch ("Orientations futures" of the MPK summary: scheduling by priority): as
 * MK_DISPATCH_CLAIM, and the critical path's tasks -- every layer's attention chunks, on which the
 * O projection of every SM waits -- are a pool too, placed right after the QKV pool in every SM's
 * queue, so the SMs that finish their QKV claims first take them instead of chunks fixed to SMs
 * that may still be streaming QKV rows. */
#define MK_DISPATCH_CLAIM_PRIORITY 3
int mk_set_dispatch(mk_ctx* ctx, int mode, int tasks_per_sm, void* stream);

/* Prefetch depth: besides the shared-memory ring (6 stages of 32 KB per SM), an SM's producer
 * that has been blocked on a full ring for over a microsecond (its workers wait for a
 * dependency, e.g. during attention) prefetches up to `stages` further weight stages of its
 * queue into L2, so HBM keeps streaming.  (Attention K/V rows are not prefetched: requesting
 * them into L2 ahead of the ring made the 16-sequence step 4 % slower on B200.)  Default 8 (measured fastest on B200, 0.7 % faster than 0 = off on the 8B batch-1 decode);
 * at most 64. */
int mk_set_l2_prefetch(mk_ctx* ctx, int stages);

/* Split-KV chunk length floor: at attention length Lk, a (sequence, KV head) uses
 * min(chunks, ceil(Lk / keys)) chunks, each on its own SM, whose partials the last one to finish
 * merges (FlashDecoding, named in the Mirage article's attention example).  Fewer, longer chunks
 * save the arrival atomic and the merge on the critical path; more, shorter ones spread the keys
 * over more SMs.  Default 64; must be in [1, 2^20].  Results do not depend on it beyond rounding. */
int mk_set_attn_chunk_keys(mk_ctx* ctx, int keys);

/* Head mode of the decode attention: while the attention length Lk is at most `keys` (and the
 * model has G > 1 query heads per KV head and at least G chunk tasks per group), chunk task
 * c < G of a (sequence, KV head) computes query head c over all Lk keys and stores its output
 * directly; no partial is written or merged, so the arrival atomic and the merge leave the
 * critical path.  Longer lengths split the keys (mk_set_attn_chunk_keys).  0 turns head mode
 * off.  Default 640; must be in [0, 2^20].  Results do not depend on it beyond rounding. */
int mk_set_attn_head_keys(mk_ctx* ctx, int keys);

/* Tracing (per-task timing of the next decode steps).  device_buffer: n_tasks * 6 uint64
 * records (n_tasks from mk_get_graph_info), or NULL to switch tracing off.  Record of task i
 * (global-timer ns): [0] worker starts waiting for the task's inputs, [1] inputs released by
 * the scheduler, [2] task done, [3] low 32 bits: worker ns blocked on weight-ring stages,
 * high 32 bits: SM, [4] producer ns blocked on a full ring while issuing the task's weight
 * stages, [5] time of the task's first weight issue.  Each step overwrites the records. */
int mk_set_trace(mk_ctx* ctx, void* device_buffer);

/* Task-graph introspection (for tests and the bench). */
typedef struct mk_graph_info {
  int n_sms;         /* workers = resident CTAs of the persistent grid */
  int n_tasks, n_events;
  int task_capacity; /* tasks the workspace can hold (re-partitioning headroom) */
  int attn_chunks;   /* split-KV chunks per (sequence, KV head) */
  int kernel_variant;/* index of the compiled instantiation chosen for this shape */
  uint64_t weight_bytes_per_step; /* bf16 weights streamed by one decode step */
  uint64_t smem_bytes;            /* dynamic shared memory per CTA */
} mk_graph_info;
int mk_get_graph_info(const mk_ctx* ctx, mk_graph_info* out);

/* Flat copy of the task graph: per task {kind, layer, sm, row0, nrows, n_wait, wait0,
 * wait1, n_notify, notify0, notify1} as 11 int32; per event its per-step count.  For an
 * attention task row0 = sequence * n_kv_heads + KV head and nrows = its split-KV chunk; for a
 * projection task of a tensor-core context (max_batch > 4) row0 = its first 128 x 128 weight
 * block (tile * K blocks + K block) and nrows = its block count; otherwise row0/nrows are
 * packed weight rows.  Returns the number of tasks (or a negative error); either buffer may
 * be NULL to query sizes. */
int mk_export_taskgraph(const mk_ctx* ctx, int32_t* tasks, int task_capacity, int32_t* event_counts,
                        int event_capacity);

/* Validate an exported-and-edited task graph with the same CPU checks mk_build_taskgraph
 * runs (used to show that corrupted graphs are rejected).  Returns MK_OK or
 * MK_ERR_INVALID_ARG with the reason in mk_last_error(ctx). */
int mk_validate_taskgraph(mk_ctx* ctx, const int32_t* tasks, int n_tasks, const int32_t* event_counts,
                          int n_events);

/* Tensor parallel (the pages' multi-GPU scheme: "Compiler des LLM en MegaKernel ...", Part 1,
 * where a matmul followed by an all-reduce is lowered into tile tasks that start the reduction
 * on partial results, and "Valeur cle de MPK", overlap of computation and communication).
 * Rank r of n_ranks holds 1/n_ranks of the query and KV heads, of the ffn rows and of the
 * vocabulary: QKV, gate/up and the LM head are split by output rows (column parallel), O and
 * down by input columns (row parallel).  Each O or down task stores its partial output rows
 * into EVERY rank's receive buffer (peer stores) and raises the op's event on every rank
 * (remote-signal edges); a rank's next op waits for all ranks' tasks and adds the ranks'
 * partials in rank order, so the replicated residual stream is bitwise the same on every rank.
 * The LM head's argmax is exchanged the same way, so every rank picks the same token.
 *
 * mk_build_taskgraph_tp builds an EMULATED tensor-parallel context: all n_ranks ranks on one
 * device, in one persistent launch of n_ranks x (SMs / n_ranks) CTAs, CTA b serving rank
 * b / (SMs / n_ranks), each rank's peer buffers in the same device memory.  Requirements:
 * n_ranks in [2, 4]; max_batch == 1; qk_norm == 0; n_kv_heads, ffn / 8 and vocab divisible by
 * n_ranks; a compiled instantiation for the shard shape (the tiny decoder over 2 ranks, the
 * Llama-3-8B shape over 2 or 4) else MK_ERR_UNSUPPORTED.  The graph of every rank is validated
 * together (mk_validate_taskgraph_tp).  The context is used with the ordinary calls:
 * mk_weight_arena_bytes / mk_workspace_bytes / mk_kv_cache_bytes (the ranks' regions one after
 * another; the cache is [rank][layer][K|V][1][n_kv_heads / n_ranks][max_seq][head_dim]),
 * mk_load_weights (the whole model's host weights; each rank's shard is cut from them),
 * mk_set_positions (a prompt is fed as decode steps from position 0, or the caller fills the
 * cache), mk_decode_step / mk_decode_steps (logits [1][vocab] whole: each rank writes its
 * vocabulary slice), mk_sync_status, mk_set_wait_timeout_ns, mk_debug_drop_notify (the event id
 * on every rank), mk_get_graph_info, mk_destroy.  mk_prefill, mk_set_sm_weights,
 * mk_set_op_sm_weights, mk_set_dispatch, mk_set_trace and mk_export_taskgraph return
 * MK_ERR_UNSUPPORTED for it. */
int mk_build_taskgraph_tp(const mk_config* cfg, int n_ranks, int device, mk_ctx** out);

/* The tensor-parallel task graph of every rank: per task 15 int32 {rank, kind, layer, sm (global:
 * rank r's SM s is r * (SMs / n_ranks) + s), row0, nrows (attention: chunk), n_wait, wait0, wait1,
 * n_notify, notify0, notify1, remote (1: the notifies go to the event on every rank), row_lo,
 * row_hi (gate/up: the rows of the residual sum x_mid this task writes; else 0)};
 * event_counts: one rank's per-step thresholds (every rank has the same).  Returns the number
 * of tasks; either buffer may be NULL to query sizes. */
int mk_export_taskgraph_tp(const mk_ctx* ctx, int32_t* tasks, int task_capacity, int32_t* event_counts,
                           int event_capacity);
/* Validate an exported-and-edited tensor-parallel graph: per rank, thresholds equal the
 * producers that reach that rank's counter (remote signals included); every op's rows,
 * attention chunks and residual rows covered once; and, with every rank's queues simulated
 * together, no deadlock and no task reading data before its producers on any rank.  MK_OK or
 * MK_ERR_INVALID_ARG with the reason in mk_last_error(ctx). */
int mk_validate_taskgraph_tp(mk_ctx* ctx, const int32_t* tasks, int n_tasks, const int32_t* event_counts,
                             int n_events);

/* Standalone decode attention in the Mirage article's example form (attention code sample:
 * Q [64,1,128], K [64,128,4096] pre-transposed, V [64,4096,128], fp16, O = softmax(Q K) V):
 *   q [BH][d], k_t [BH][d][L] (key index fastest), v [BH][L][d]: fp16 device arrays;
 *   o [BH][d]: fp32 device output; o[h] = sum_j softmax_j(scale * q[h].k_t[h][:,j]) v[h][j].
 * Accumulation and softmax in fp32, split-KV over all SMs with an online-softmax merge.
 * d must be 64 or 128; L >= 1; scale = 1.0 reproduces the example (no scaling).
 * workspace: device scratch of mk_attention_workspace_bytes(BH, d, L) bytes, 256-byte
 * aligned; its counter words must be zero before the first call (e.g. cudaMemset once);
 * every call leaves them zero again.  Calls sharing a workspace must not overlap. */
size_t mk_attention_workspace_bytes(int BH, int d, int L);
int mk_attention_decode(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d, int L,
                        float scale, void* workspace, void* stream);
/* Synchronise `stream` and report whether an mk_attention_decode call with these sizes
 * and this workspace had a device wait run out (MK_ERR_DEVICE_TIMEOUT; the workspace is
 * then re-zeroed) or finished normally (MK_OK). */
int mk_attention_status(void* workspace, int BH, int d, int L, void* stream);

/* mk_attention_decode without a workspace argument, for callers that may not allocate device
 * memory: e.g. a serving process whose own allocator reserved the GPU's memory up front, or a
 * latency-critical loop where cudaMalloc / cudaFree would block and synchronise the device.
 * (No counterpart in the pages: an addition for such callers.)  Same operands, layouts,
 * arithmetic and result as mk_attention_decode; the scratch is a fixed 4 MiB array inside
 * the library that every GPU loading the library keeps until the process exits.  Sizes whose
 * scratch (mk_attention_workspace_bytes(BH, d, L)) exceeds 4 MiB are rejected with
 * MK_ERR_INVALID_ARG and a message; a device index of 64 or more with MK_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address (once, with that device
 * current); make that first call before any stream capture.  The call allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine); it zeroes the array's arrival counts on
 * `stream` before the kernel.  A device wait that runs out is recorded in an error word at the
 * end of the array, which keeps the first such event until mk_attention_noalloc_status reads
 * it.  All calls share the one array, so calls that overlap on the GPU (other streams, other
 * threads) race: order them on one stream. */
int mk_attention_decode_noalloc(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d,
                                int L, float scale, void* stream);
/* Synchronise `stream` and report whether any mk_attention_decode_noalloc call on the current
 * device since the previous mk_attention_noalloc_status had a device wait run out
 * (MK_ERR_DEVICE_TIMEOUT: that call's output is undefined; the error word is cleared) or not
 * (MK_OK).  Allocates nothing: the word is read and cleared with cudaMemcpyFromSymbol /
 * cudaMemcpyToSymbol of 4 bytes. */
int mk_attention_noalloc_status(void* stream);

/* Limit, in nanoseconds, of every device-side wait of mk_attention_decode and
 * mk_attention_decode_noalloc calls issued after this one (process-wide; default 2e9).  Must
 * be > 0. */
int mk_attention_set_wait_timeout_ns(uint64_t ns);
/* Test hook for failure detection (process-wide): while unit >= 0, the split-KV attention
 * kernels launched afterwards never load the 64-key unit with that global index (head h's units
 * are h * ceil(L/64) ..), so the compute warp waiting for it runs out of time and the call's
 * status reports MK_ERR_DEVICE_TIMEOUT.  Nothing faults or traps.  unit < 0 switches it off. */
int mk_attention_debug_drop_unit(int unit);

/* Last error text for ctx (or the thread's last context-free error when ctx is NULL). */
const char* mk_last_error(const mk_ctx* ctx);
void mk_destroy(mk_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
