// mk_internal.h -- structures shared by the library's host code and its kernels.
//
// Task graph (Part 1 "Compilateur" of the MPK summary "Compiler des LLM en MegaKernel ..."):
// a task is one tile of one op assigned to one SM (worker); an event is a counter in device
// memory with a per-step threshold.  A task waits on up to two events and notifies up to
// two.  Thresholds are epoch-based: during decode step e (1, 2, ...) event v is active once
// its counter reaches e * count[v], so nothing is reset between steps.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "mk.h"

namespace mk {

// ---- persistent decode kernel geometry ----
#ifndef MK_WORKER_WARPS
#define MK_WORKER_WARPS 8
#endif
constexpr int kWorkerWarps = MK_WORKER_WARPS;        // compute role (the "worker" of Part 2)
constexpr int kAttnWarps = 8;                        // workers that walk keys in an attention task
constexpr int kWorkerThreads = kWorkerWarps * 32;    // 256
constexpr int kProducerWarp = kWorkerWarps;          // TMA weight streaming
constexpr int kSchedWarp = kWorkerWarps + 1;         // event polling (the "scheduler" role)
constexpr int kBlockThreads = (kWorkerWarps + 2) * 32;
constexpr int kIssuerWarp = kWorkerWarps + 2;        // tensor-core kernel: tcgen05.mma issue
constexpr int kTcBlockThreads = (kWorkerWarps + 3) * 32;
constexpr int kSegElems = kWorkerThreads * 8;        // K elements one pass of all workers covers
constexpr int kSegBytes = kSegElems * 2;
constexpr int kTaskRows = 256;                       // rows per GEMV task (one per worker thread)
constexpr int kRpsMax = 8;                           // rows per ring stage (unrolled in the GEMV loop)
constexpr int kMaxChunks = 64;                       // split-KV chunks per (sequence, KV head)
constexpr int kMaxTpRanks = 4;                       // tensor-parallel ranks one launch can host
#ifndef MK_SLOT_KB
#define MK_SLOT_KB 32
#endif
#ifndef MK_STAGES
#define MK_STAGES 6
#endif
constexpr int kSlotBytes = MK_SLOT_KB * 1024;        // one ring stage
constexpr int kStages = MK_STAGES;                   // ring depth (kStages x kSlotBytes per SM)
constexpr int kMaxDecodeBatch = 4;                   // CUDA-core path: batch width 1 or 4
constexpr int kDownChunk = 4096;                     // down-projection K chunk for batch width 4
// Tensor-core projection tiles (batch width 5..16): a tile is kTcRows weight rows; a ring
// stage is one block of kTcRows x kTcUnitK bf16 weights in the no-swizzle K-major core-matrix
// layout; a task covers up to kTcUnitsMax blocks (K units) of one tile.  Activations are
// staged kTcSegUnits units at a time into one of two operand buffers.
constexpr int kTcBatch = 16;                         // sequences per tensor-core step (MMA N = 2 x 16)
constexpr int kTcN = 2 * kTcBatch;                   // columns: bf16 high parts, then low parts
constexpr int kTcRows = 128;                         // MMA M
constexpr int kTcUnitK = 128;                        // K elements per ring stage
constexpr int kTcUnitsMax = 64;                      // K units per task
constexpr int kTcSegUnits = 4;                       // K units per activation segment
constexpr int kTcStages = 4;                         // ring depth of the tensor-core kernel
constexpr int kTcBopSbo = kTcSegUnits * kTcUnitK / 8 * 128;  // operand buffer: bytes per 8-row group
constexpr int kTcBopBuf = (kTcN / 8) * kTcBopSbo;   // one operand buffer (32 KB)
constexpr int kTcBopBytes = 2 * kTcBopBuf;          // two buffers
constexpr int kTcRecFloats = kTcRows * kTcBatch + kTcBatch;  // partial record: [row][seq] sums, seq sum of x^2
static_assert(kTcRows * kTcUnitK * 2 == MK_SLOT_KB * 1024, "a weight block fills one ring stage");

enum TaskKind : uint8_t {
  TK_EMBED = 1,   // x_0 = E[token] for a slice of rows
  TK_QKV = 2,     // q,k,v rows of W_qkv . RMSNorm(x); RoPE; K/V append
  TK_ATTN = 3,    // split-KV chunk of one (sequence, KV head); last arriver merges
  TK_OPROJ = 4,   // x_mid = x + W_o o
  TK_GATEUP = 5,  // h = silu(W_g xn) * (W_u xn), rows interleaved (g_i, u_i)
  TK_DOWN = 6,    // x_next = x_mid + W_d h
  TK_LMHEAD = 7,  // logits rows of W_lm . RMSNorm(x); per-task argmax partial
  TK_POOL = 8,    // queue entry (run-time claims): claim tasks of pool `index` until it is empty
};

struct Task {
  uint8_t kind, n_wait, n_notify, pad0;
  uint16_t layer, aux;  // ATTN: aux = chunk index
  uint32_t row0;        // GEMV: first (packed) row; ATTN: b * n_kv_heads + kv head; EMBED: first row
  uint32_t nrows;       // GEMV / EMBED: row count; ATTN: 0
  uint32_t wait[2];
  uint32_t notify[2];   // ATTN: notify[0] is raised by the merging (last) chunk only
  uint32_t index;       // LMHEAD: ordinal among LM-head tasks (argmax partial slot)
  uint32_t pad1;
  // Tensor-parallel graphs: pad0 = 1 marks a remote-signal edge (the task's notifies go to the
  // event of that id on every rank); gate/up tasks also write the rows [index, pad1) of the
  // residual sum x_mid they form (each rank keeps its copy, shared out over its tasks).
  // Tensor-core tasks reuse the fields: row0 = first weight block (tile * K units + unit),
  // nrows = blocks, index = partial record, aux = slot among the tile's tasks (the tile's
  // records are index - aux ..), pad0 = tasks of the tile, pad1 = tile arrival counter.
};
static_assert(sizeof(Task) == 40, "Task layout");

// Byte offsets of one layer's tensors in the weight arena.
struct LayerOff {
  uint64_t qkv, o, gu, d;   // packed matrices
  uint64_t attn_norm, mlp_norm;
  uint64_t qkn;             // QK-norm: q gain [nq*D], q bias [nq*D], k gain [nkv*D], k bias [nkv*D]
};

struct DecodeParams {
  const Task* tasks;
  const uint32_t* qbegin;     // [n_sms + 1]
  const uint32_t* ev_count;   // [n_events]
  uint32_t* ev;               // [n_events] counters
  uint32_t* acnt;             // [L][B][nkv] attention chunk arrivals
  uint32_t* err;              // [4]: code, where, task, global abort flag
  const uint8_t* arena;
  const LayerOff* loff;       // [L]
  uint64_t off_embed, off_lm, off_fnorm;
  const float2* rope;         // [max_seq][D/2] (cos, sin)
  uint16_t* kv;               // [L][2][max_batch][nkv][max_seq][D]
  float* x_in;                // [L+1][B][H]
  float* x_mid;               // [L][B][H]
  float* qbuf;                // [L][B][nq*D] (QK-norm: before the norm and RoPE)
  float* kraw;                // QK-norm: [L][B][nkv*D] k before the norm and RoPE
  float* obuf;                // [L][B][nq*D]
  float* hbuf;                // [L][B][F]
  float* part;                // [L][B][nq][nch][D+2]
  float* lm_val;              // [n_lm][B]
  int32_t* lm_idx;            // [n_lm][B]
  const int32_t* tokens;      // [B]
  float* logits;              // [B][V]
  int32_t* next_tokens;       // [n_steps][B] greedy tokens of every step (null: not kept, 1 step only)
  int pos[MK_MAX_BATCH];
  int B, H, nq, nkv, D, F, V, L, nch, max_seq, max_batch, n_lm;
  float eps, attn_scale;
  uint32_t epoch;
  uint32_t ev_lm;             // event counting finished LM-head tasks (last one picks the token)
  int drop_event;             // test hook: notify skipped for this event id (-1 = none)
  uint64_t timeout_ns;
  uint64_t* trace;            // optional [n_tasks][kTraceWords] timing records (null = off)
  int l2_ahead;               // weight stages the producer prefetches into L2 beyond the ring
  int min_chunk_keys;         // split-KV: a chunk in use holds at least this many keys
  int head_keys;              // up to this attention length a chunk takes one query head, no merge
  int nb;                     // active sequences (<= the kernel's batch width)
  int kdc, ndc;               // down-projection K chunk and chunk count
  float* tpart;               // tensor-core partial records [n_records][kTcRecFloats]
  uint32_t* tcnt;             // tensor-core tile arrival counters
  int n_steps;                // greedy decode steps in this launch (step s: epoch + s, pos + s)
  uint32_t ev_tok;            // event: the step's tokens are picked (the next step's embedding waits)
  int qk_norm;                // 1: LayerNorm of every q and k head before RoPE, in the attention task
  // run-time claims: pools[p] = (first task, task count); pcnt[4][n_pools] claim counters, one
  // row per step (epoch mod 4), the row of step e + 2 zeroed by step e's token pick
  const uint2* pools;
  uint32_t* pcnt;
  int n_pools;
  int dyn;
  // Tensor parallel (the TP instantiation only; "Compiler des LLM en MegaKernel ...", Part 1:
  // a matmul followed by an all-reduce lowered into tile tasks).  This view is rank tp_rank of
  // tp_ranks; its weights, KV cache and activations are its shard.  The row-parallel O and down
  // tasks store their partial rows into EVERY rank's receive buffer (peer stores) and raise the
  // op's event on every rank (remote signals); consumers add the ranks' partials in rank order,
  // so the replicated residual stream is bitwise the same on every rank.  Only x_mid[l] is
  // stored (by the gate/up tasks); QKV, gate/up and the LM head form x_in[l] = x_mid[l-1] +
  // the ranks' down rows of layer l-1 as they load it.
  int tp_rank, tp_ranks;
  int tp_vbase, tp_vfull;          // LM head: this rank's first vocab row; the full vocab (logits stride)
  float* tp_recv_o[kMaxTpRanks];   // rank d's O-projection receive buffer [L][ranks][B][H]
  float* tp_recv_d[kMaxTpRanks];   // rank d's down-projection receive buffer [L][ranks][B][H]
  uint32_t* tp_ev[kMaxTpRanks];    // rank d's event counters
  uint64_t* tp_lmx[kMaxTpRanks];   // rank d's argmax slots [ranks][B]: value bits << 32 | vocab index
  uint32_t ev_lmx;                 // event: every rank's argmax partial of the step arrived
};

// One launch hosting several tensor-parallel ranks on one GPU (CTA b serves rank
// b / sms_per_rank): the ranks' views, each pointing at its own shard.
struct DecodeParamsTP {
  DecodeParams r[kMaxTpRanks];
  int sms_per_rank;
};
constexpr int kDynQ = 64;                 // run-time claims: task FIFO from the producer to the other roles
constexpr uint32_t kDynEnd = 0xffffffffu;  // FIFO entry: no more tasks in this launch
constexpr uint64_t kStallPrefetchNs = 1000;    // producer blocked this long: prefetch ahead into L2
constexpr uint64_t kStallPrefetchGapNs = 100;   // then one more stage per this interval
constexpr int kTcMinBatchDefault = 2;    // max_batch from which the tensor-core instantiation runs
constexpr int kHeadKeysDefault = 640;     // head-mode attention up to this length (mk_set_attn_head_keys)
constexpr int kMinChunkKeysDefault = 64;  // split-KV chunks hold at least this many keys (mk_set_attn_chunk_keys)

// Trace record per task (global-timer ns): worker start of the wait for inputs, inputs
// released, task done; worker ns blocked on ring stages | SM id << 32; producer ns blocked
// on a full ring while issuing this task's stages; producer time of the task's first issue.
constexpr int kTraceWords = 6;

// Error word layout in the workspace.
enum { ERR_CODE = 0, ERR_WHERE = 1, ERR_TASK = 2, ERR_ABORT = 3 };
enum { DEV_ERR_WAIT_EVENT = 1, DEV_ERR_WAIT_READY = 2, DEV_ERR_WAIT_FULL = 3, DEV_ERR_WAIT_EMPTY = 4,
       DEV_ERR_BAD_TOKEN = 5 };

typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeFn get_tensor_map_encoder();

// Kernel variants: one instantiation per (segments, rows per stage) of the two K sizes.
struct Variant {
  int nseg_h, rps_h, nseg_f, rps_f, head_dim, bm, qkn, dyn, tp;
};
int find_decode_variant(int nseg_h, int rps_h, int nseg_f, int rps_f, int head_dim, int bm, int qkn, int dyn,
                        int tp = 0);
const void* decode_kernel_ptr(int variant);
size_t decode_smem_bytes(int variant);
int launch_decode(int variant, const DecodeParams& p, int grid, cudaStream_t stream, std::string* err);
// The tensor-parallel instantiation: n_ranks views, grid = n_ranks * sms_per_rank CTAs.
int launch_decode_tp(int variant, const DecodeParams* views, int n_ranks, int sms_per_rank, cudaStream_t stream,
                     std::string* err);

// Standalone attention (mk_attention.cu).  err_word: where the kernel records a wait that
// ran out (null: the workspace's own error word).  The wait limit and the drop-unit test hook
// are process-wide settings.
size_t attention_workspace_bytes(int BH, int d, int L, int n_sms);
size_t attention_error_word_offset(int BH, int d, int L, int n_sms);
int attention_decode(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d, int L,
                     float scale, void* workspace, cudaStream_t stream, int n_sms, uint32_t* err_word,
                     std::string* err);
size_t attention_counter_offset(int BH, int d, int L, int n_sms);
size_t attention_noalloc_capacity();
int attention_decode_noalloc(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d,
                             int L, float scale, cudaStream_t stream, std::string* err);
int attention_noalloc_status(cudaStream_t stream, std::string* err);
void attention_set_wait_timeout_ns(uint64_t ns);
void attention_debug_drop_unit(int unit);

// Prefill (mk_prefill.cu).
struct PrefillParams {
  const uint8_t* arena;
  const LayerOff* loff_host;  // host copy of per-layer offsets
  uint64_t off_embed, off_lm, off_fnorm;
  const float2* rope;
  uint16_t* kv;
  float *X, *XN, *Y, *Q, *O, *HH;  // scratch [rows][...]
  int rows_cap;
  int H, nq, nkv, D, F, V, L, max_seq, max_batch;
  float eps, attn_scale;
  int kdc, ndc;  // W_down stored in ndc chunk-major K chunks of kdc columns
  int blocked;   // 1: projections in the tensor-core block layout (kTcRows x kTcUnitK blocks)
  int qk_norm;   // 1: LayerNorm of every q and k head before RoPE
};
int run_prefill(const PrefillParams& p, const int32_t* tokens, int B, int T, float* last_logits,
                cudaStream_t stream, std::string* err);

}  // namespace mk
