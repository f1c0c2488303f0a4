// mk_decode.cu -- the persistent decode megakernel (one launch per decode step).
//
// Runtime of the MPK summary "Compiler des LLM en MegaKernel ..." Part 2 "Runtime":
// one CTA per SM runs the tasks of its queue in order ("Workers": fetch, execute, notify,
// repeat); a scheduler role watches the event counters ("Schedulers", "Execution pilotee
// par evenements": a finished task increments an event counter; once the counter reaches
// its threshold the dependent tasks may run).  Roles inside each CTA:
//   warps 0-7  worker:    GEMV / attention / epilogues of the current task
//   warp 8     producer:  streams the queue's weight tiles into a 6-stage shared-memory ring
//                         with 1-D TMA bulk copies; weights never depend on activations, so
//                         it runs ahead across dependency waits (the cross-layer overlap of
//                         the same summary's "Valeur cle" / Part 2)
//   warp 9     scheduler: acquires the events the next tasks wait on and releases them to the
//                         workers through a shared-memory counter
// Every wait is bounded by a global-timer limit; a wait that runs out records an error word,
// raises a global abort flag that every CTA polls, and all roles return (the producer first
// waits, bounded, for its copies in flight).
//
// GEMV tiles: a task is up to 32 rows x full K.  Each of the 256 worker threads owns 8 K
// elements of every 2048-element segment, so x (times the norm gain) sits in registers for
// the whole task and each weight byte is read from shared memory once; partial sums are
// reduced across lanes with a transposed butterfly of shuffles (lane r ends with row r) and
// across warps through shared memory.  RMSNorm is fused by the "Normalization + Linear"
// identity of the Mirage article (Case 1): dot(W, x*g) * rsqrt(mean(x^2) + eps).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cstring>

#include "mk_internal.h"
#include "mk_ptx.cuh"

namespace mk {

// Dynamic shared memory: the weight ring (nst stages of kSlotBytes, 1024-aligned), then for
// the tensor-core kernel the activation operand (kTcBopBytes), then DSmem.
struct DSmem {
  union {
    float red[kWorkerWarps][kTaskRows];  // GEMV: per-warp sums of the current task, [row][seq]
    float aacc[kAttnWarps][4][128];      // attention: per-warp partial outputs
    float tile[kTcRecFloats];            // tensor-core tile: summed partial records
    float wp[kAttnWarps][512];           // wide attention: a warp's probabilities [head][key] (warp w
                                         // uses only row w, which its own aacc row overlays)
  };
  float tot[kTaskRows];                  // totals of the current task, [row][seq]
  float ssw[kWorkerWarps][kMaxDecodeBatch];  // per-warp sums of x^2 per sequence
  float am[kAttnWarps][4];
  float al[kAttnWarps][4];
  union {
    struct {
      float mm[4 * kMaxChunks], ll[4 * kMaxChunks];  // split-KV merge of the last arriver (after the key loop)
    } mg;
    float qn[4 * 128];  // QK-norm: an attention task's normed, rotated q heads (read before its key loop)
  };
  float lmv[kWorkerWarps];
  int lmi[kWorkerWarps];
  float tss[2][kTcBatch];    // tensor-core tasks (by parity): per-sequence sum of x^2 over the K range
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t bop_full[2];      // tensor-core operand buffer staged (one arrival per worker warp)
  uint64_t bop_free[2];      // ... and read by its MMAs (tcgen05.commit)
  uint64_t acc_full[2];      // tensor-core accumulator complete (tcgen05.commit)
  uint64_t acc_free[2];      // ... and read back (one arrival per reading warp)
  uint64_t mma_done;         // every MMA issued so far completed (issuer drain at exit)
  uint64_t kv_full[2];       // tensor-core attention: K/V stage loaded into operand buffer b
  uint64_t kv_empty[2];      // ... and read by both warps of the last warp pair
  uint32_t tmem;             // tensor-memory accumulators (2 x kTcN columns)
  uint32_t ready;            // tasks [0, ready) of this queue have their inputs
  // ring stage s holds the stage with this launch-wide sequence number (published by the
  // producer once armed): a warp that takes stages out of order (wide attention) first waits
  // for its stage's number, so a parity wait is never a phase ahead
  uint32_t armed[kStages];
  uint32_t cabort;           // worker-role abort: written before, read after a worker barrier
  volatile uint32_t abort;   // any role gave up: stop waiting
  uint32_t flag;             // worker broadcast (last-arriver decisions)
  // run-time claims: task FIFO from the producer (which claims) to the scheduler and workers
  uint32_t dq_id[kDynQ];
  uint16_t dq_st[kDynQ];
  uint32_t dq_n;             // entries pushed
  uint32_t wdone;            // entries the workers finished (their slots can be reused)
};

__host__ __device__ constexpr int ring_stages(bool tc) { return tc ? kTcStages : kStages; }
__host__ __device__ constexpr size_t ring_bytes(bool tc) {
  return (size_t)ring_stages(tc) * kSlotBytes + (tc ? (size_t)kTcBopBytes : 0);
}

static_assert(ring_bytes(false) + sizeof(DSmem) + 1024 <= 227 * 1024 &&
                  ring_bytes(true) + sizeof(DSmem) + 1024 <= 227 * 1024,
              "dynamic shared memory of a CTA exceeds 227 KB");

__device__ __forceinline__ void worker_bar() { named_bar_sync(1, kWorkerThreads); }

__device__ __forceinline__ void raise_error(const DecodeParams& P, DSmem& S, uint32_t code, uint32_t where,
                                            uint32_t task) {
  S.abort = 1u;
  if (atomicCAS(&P.err[ERR_CODE], 0u, code) == 0u) {
    P.err[ERR_WHERE] = where;
    P.err[ERR_TASK] = task;
  }
  atomicExch(&P.err[ERR_ABORT], 1u);
}

// Bounded mbarrier wait (see header comment).  False once the limit passed or a role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns, DSmem* S) {
  if (mbar_test_now(bar, parity)) return true;  // common case: already complete
  uint64_t t0 = 0;
  for (uint32_t n = 1;; ++n) {
    if (mbar_test(bar, parity)) return true;
    if ((n & 127u) == 0) {
      if (S && S->abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) return false;
    }
  }
}

struct Pipe {
  int stage;
  uint32_t phase;
  int nst;       // ring depth
  uint32_t seq;  // launch-wide number of the next stage
  __device__ __forceinline__ void advance() {
    ++seq;
    if (++stage == nst) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// acc (even/odd partial sums packed in one register pair) += the 8 bf16 weights of w times
// the packed x pairs: each 32-bit word holds weights (2j, 2j+1) and meets x pair j.
__device__ __forceinline__ void dot8(const uint4 w, const uint64_t* x2, uint64_t& acc) {
  fma2_bf16w(acc, w.x, x2[0]);
  fma2_bf16w(acc, w.y, x2[1]);
  fma2_bf16w(acc, w.z, x2[2]);
  fma2_bf16w(acc, w.w, x2[3]);
}

__device__ __forceinline__ uint16_t f2bf(float f) {
  // round to nearest even
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float bf2f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// Which stream a GEMV task reads: arena offset and row length (bytes) for the task's op.  A
// tensor-core task streams whole weight blocks: row0 counts blocks of kSlotBytes.
template <bool TC>
__device__ __forceinline__ void gemv_source(const DecodeParams& P, const Task& t, uint64_t* off, uint32_t* row_bytes) {
  const LayerOff& lo = P.loff[t.layer < P.L ? t.layer : 0];
  if (TC) {
    switch (t.kind) {
      case TK_QKV: *off = lo.qkv; break;
      case TK_OPROJ: *off = lo.o; break;
      case TK_GATEUP: *off = lo.gu; break;
      case TK_DOWN: *off = lo.d; break;
      default: *off = P.off_lm; break;
    }
    *row_bytes = (uint32_t)kSlotBytes;
    return;
  }
  switch (t.kind) {
    case TK_QKV: *off = lo.qkv; *row_bytes = (uint32_t)P.H * 2u; break;
    case TK_OPROJ: *off = lo.o; *row_bytes = (uint32_t)(P.nq * P.D) * 2u; break;  // K = the heads' width
    case TK_GATEUP: *off = lo.gu; *row_bytes = (uint32_t)P.H * 2u; break;
    case TK_DOWN: {  // K chunk t.aux of W_down: chunk-major, rows of kc = min(kdc, F - k0) weights
      const uint32_t k0 = (uint32_t)t.aux * (uint32_t)P.kdc;
      const uint32_t kc = min((uint32_t)P.kdc, (uint32_t)P.F - k0);
      *off = lo.d + (uint64_t)k0 * P.H * 2u;
      *row_bytes = kc * 2u;
      break;
    }
    default: *off = P.off_lm; *row_bytes = (uint32_t)P.H * 2u; break;
  }
}

__device__ __forceinline__ bool is_gemv(uint8_t k) {
  return k == TK_QKV || k == TK_OPROJ || k == TK_GATEUP || k == TK_DOWN || k == TK_LMHEAD;
}

// ---------------------------------------------------------------------------------------
// Warp reduction of the V (power of two) row partials a[0..V) of one ring stage: transposed
// butterfly (each exchange halves the live values), then a plain butterfly over the lanes
// left; lane l with l % (32/V) == 0 ends with the warp's sum for row r(l).
__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

template <int V>
__device__ __forceinline__ void warp_reduce_rows(float (&a)[V], float* out, int lane, int valid) {
  constexpr int LV = ilog2(V);
#pragma unroll
  for (int k = 0; k < LV; ++k) {
    const int off = 16 >> k, half = (V >> k) >> 1;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? a[i] : a[i + half];
      const float keep = upper ? a[i + half] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 >> LV; off >= 1; off >>= 1) a[0] += __shfl_xor_sync(0xffffffffu, a[0], off);
  if ((lane & ((32 >> LV) - 1)) == 0) {
    int r = 0;
#pragma unroll
    for (int k = 0; k < LV; ++k) r += ((lane >> (4 - k)) & 1) * ((V >> k) >> 1);
    if (r < valid) out[r] = a[0];
  }
}

// GEMV core: tot[r * BM + b] = sum_k W[row0 + r][k] * x_b[k] * g[k] for r < nrows and the
// nb (<= BM) sequences b, where x_b = xsrc + b * xstride; nrows * BM <= kTaskRows.  Rows are
// streamed through the ring RPS rows per stage, so each weight is read from shared memory
// once and meets all BM activation vectors.  The stage loop is a runtime loop and only one
// stage's rows are unrolled, so the code stays small; each stage's RPS x BM sums are reduced
// across lanes right away into S.red[warp][row * BM + b], and across warps at the end into
// S.tot.  Also leaves the per-warp sums of x_b^2 in S.ssw for the fused norm.  Returns false
// (for every worker thread alike) if a wait ran out.
// Tensor-parallel input of a GEMV: x = xsrc + add[0] + add[stride] + ... (n ranks' partial
// rows) + add2[0] + add2[stride] + ... (n2 more), added in that order so every rank gets the
// same bits; the sum's elements [mlo, mhi) (multiples of 8) are also stored to mat.
struct XAdd {
  const float* add;
  int n;
  const float* add2;
  int n2;
  size_t stride;
  float* mat;
  int mlo, mhi;
};

template <int NSEG, int RPS, int BM, bool TPX = false>
__device__ __forceinline__ bool gemv_tile(const DecodeParams& P, DSmem& S, Pipe& pp, const uint8_t* ring,
                                          const float* __restrict__ xsrc,
                                          int xstride, int nb, const uint16_t* __restrict__ gain, int K, int nrows,
                                          uint32_t row_bytes, uint32_t task_id, uint32_t& stall_ns,
                                          const XAdd& xa = XAdd{nullptr, 0, nullptr, 0, 0, nullptr, 0, 0}) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // only the last segment can be partial or empty: K > (NSEG - 2) * kSegElems by construction,
  // except in a tensor-parallel shard, where the O projection's K (the rank's heads) can end
  // inside an earlier segment: there every segment is checked
  const bool last_ok = (NSEG - 1) * kSegElems + tid * 8 < K;
  auto seg_ok = [&](int s) { return TPX ? (s * kSegElems + tid * 8 < K) : (s < NSEG - 1 || last_ok); };
  uint64_t x2[BM][NSEG][4];
  float ss[BM];
#pragma unroll
  for (int b = 0; b < BM; ++b) {
    ss[b] = 0.f;
#pragma unroll
    for (int s = 0; s < NSEG; ++s) {
      const int k = s * kSegElems + tid * 8;
      float x[8];
      if (seg_ok(s) && (BM == 1 || b < nb)) {
        const float* xb = xsrc + (size_t)b * xstride;
        float4 a = ldcg_f4(xb + k);
        float4 c = ldcg_f4(xb + k + 4);
        if constexpr (TPX) {
          for (int r = 0; r < xa.n + xa.n2; ++r) {
            const float* ad = (r < xa.n ? xa.add + (size_t)r * xa.stride : xa.add2 + (size_t)(r - xa.n) * xa.stride) + k;
            const float4 u = ldcg_f4(ad);
            const float4 w = ldcg_f4(ad + 4);
            a.x += u.x; a.y += u.y; a.z += u.z; a.w += u.w;
            c.x += w.x; c.y += w.y; c.z += w.z; c.w += w.w;
          }
          if (xa.mat && k >= xa.mlo && k < xa.mhi) {
            *reinterpret_cast<float4*>(xa.mat + k) = a;
            *reinterpret_cast<float4*>(xa.mat + k + 4) = c;
          }
        }
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss[b] = fmaf(x[i], x[i], ss[b]);
        if (gain) {
          const uint4 g = __ldg(reinterpret_cast<const uint4*>(gain + k));
          x[0] *= bf16lo(g.x); x[1] *= bf16hi(g.x);
          x[2] *= bf16lo(g.y); x[3] *= bf16hi(g.y);
          x[4] *= bf16lo(g.z); x[5] *= bf16hi(g.z);
          x[6] *= bf16lo(g.w); x[7] *= bf16hi(g.w);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) x2[b][s][j] = pack2(x[2 * j], x[2 * j + 1]);
    }
  }
  // the per-warp sums of x^2 for the fused norm, stored before the stage loop so that they do
  // not stay live across it (read after the task's last worker barrier)
#pragma unroll
  for (int b = 0; b < BM; ++b) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss[b] += __shfl_xor_sync(0xffffffffu, ss[b], off);
    if (lane == 0) S.ssw[warp][b] = ss[b];
  }
  float* red = S.red[warp];
  bool ok = true;
  for (int r0 = 0; r0 < nrows; r0 += RPS) {
    const uint64_t tw = (P.trace && tid == 0) ? globaltimer_ns() : 0;
    if (!wait_bar(&S.full[pp.stage], pp.phase, P.timeout_ns, &S)) {
      if (ok) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
      ok = false;
      S.cabort = 1u;
    }
    if (P.trace && tid == 0) stall_ns += (uint32_t)(globaltimer_ns() - tw);
    const uint8_t* base = ring + (size_t)pp.stage * kSlotBytes + tid * 16;
    // rows in sub-blocks of RSUB (all of the stage's rows at batch width 1; two at width 4,
    // which keeps 8 accumulator pairs live instead of 16)
    constexpr int RSUB = (BM == 1) ? RPS : ((8 / BM) < RPS ? (8 / BM) : RPS);
#pragma unroll
    for (int rs = 0; rs < RPS; rs += RSUB) {
      uint64_t acc[RSUB][BM];  // per (row, sequence): (even, odd) partial sums
#pragma unroll
      for (int rr = 0; rr < RSUB; ++rr) {
#pragma unroll
        for (int b = 0; b < BM; ++b) acc[rr][b] = 0ull;
        if (RPS == 1 || r0 + rs + rr < nrows) {
#pragma unroll
          for (int s = 0; s < NSEG; ++s) {
            if (seg_ok(s)) {
              const uint4 w = *reinterpret_cast<const uint4*>(base + (rs + rr) * row_bytes + s * kSegBytes);
              if (BM == 1) {
                dot8(w, x2[0][s], acc[rr][0]);
              } else {
                const uint64_t wp[4] = {widen_bf16w(w.x), widen_bf16w(w.y), widen_bf16w(w.z), widen_bf16w(w.w)};
                // sequences innermost: consecutive FMAs update different accumulators
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                  for (int b = 0; b < BM; ++b)
                    if (b < nb) fma2_pair(acc[rr][b], wp[j], x2[b][s][j]);
              }
            }
          }
        }
      }
      if (rs + RSUB >= RPS) {  // the stage's last shared-memory read is done: release it
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[pp.stage]);
      }
      float a[RSUB * BM];
#pragma unroll
      for (int rr = 0; rr < RSUB; ++rr)
#pragma unroll
        for (int b = 0; b < BM; ++b) {
          const float2 v = unpack2(acc[rr][b]);
          a[rr * BM + b] = v.x + v.y;
        }
      warp_reduce_rows<RSUB * BM>(a, red + (r0 + rs) * BM, lane, (nrows - r0 - rs) * BM);
    }
    pp.advance();
  }
  worker_bar();
  if (S.cabort) return false;
  for (int t = tid; t < nrows * BM; t += kWorkerThreads) {
    float v = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kWorkerWarps; ++w2) v += S.red[w2][t];
    S.tot[t] = v;
  }
  worker_bar();
  return true;
}

__device__ __forceinline__ float norm_factor(const DSmem& S, int K, float eps, int b) {
  float ss = 0.f;
#pragma unroll
  for (int w = 0; w < kWorkerWarps; ++w) ss += S.ssw[w][b];
  return 1.0f / sqrtf(ss / (float)K + eps);
}

// ---------------------------------------------------------------------------------------
// Epilogues: thread e < nrows * BM handles row row0 + e / BM of sequence b = e % BM, whose
// GEMV total is S.tot[e] (sequences b >= nb are skipped).
// Packed QKV row R of sequence b (value v; other = its RoPE partner row R ^ 1): q rows go to
// qbuf after RoPE, k rows after RoPE and v rows as they are into the bf16 cache at pos[b].
// With QK-norm the q and k rows are stored as they are (qbuf, kraw; natural dim order): the
// LayerNorm needs a whole head, which the attention task of its KV head holds, so the norm
// and RoPE of q and of the new key happen there.
// RoPE angle (cos, sin) that packed QKV row R of sequence b takes at step st: (1, 0) for v rows
// and with QK-norm (whose RoPE runs in the attention task).  A constant table: callers may load
// it before the task's inputs exist.
__device__ __forceinline__ float2 qkv_rope_angle(const DecodeParams& P, int R, int b, int st) {
  const int D = P.D, G = P.nq / P.nkv;
  const int rr = R % ((G + 2) * D);
  if (P.qk_norm || rr >= (G + 1) * D) return make_float2(1.f, 0.f);
  const int pd = (rr < G * D) ? (rr % D) : (rr - G * D);
  return __ldg(P.rope + (size_t)(P.pos[b] + st) * (D / 2) + (pd >> 1));
}

__device__ __forceinline__ void qkv_out(const DecodeParams& P, int layer, int R, int b, float v, float other,
                                        int st, float2 cs) {
  const int D = P.D, G = P.nq / P.nkv, half = D / 2;
  const int rpg = (G + 2) * D;
  const int grp = R / rpg, rr = R % rpg;
  const int pos = P.pos[b] + st;  // step st of the launch
  const size_t head_stride = (size_t)P.max_seq * D;
  const size_t kv_layer = (size_t)P.max_batch * P.nkv * head_stride;  // one of K or V, one layer
  if (rr < (G + 1) * D) {
    // q or k: rows come in RoPE pairs (i, i + D/2) at packed positions (2i, 2i+1)
    const int pd = (rr < G * D) ? (rr % D) : (rr - G * D);
    const int i = pd >> 1, hi = pd & 1;
    if (P.qk_norm) {
      const int dim = hi ? i + half : i;
      if (rr < G * D)
        P.qbuf[((size_t)layer * P.B + b) * P.nq * D + (size_t)(grp * G + rr / D) * D + dim] = v;
      else
        P.kraw[((size_t)layer * P.B + b) * P.nkv * D + (size_t)grp * D + dim] = v;
      return;
    }
    float outv;
    int dim;
    if (hi == 0) {
      outv = v * cs.x - other * cs.y;
      dim = i;
    } else {
      outv = v * cs.x + other * cs.y;
      dim = i + half;
    }
    if (rr < G * D) {
      const int hq = grp * G + rr / D;
      P.qbuf[((size_t)layer * P.B + b) * P.nq * D + (size_t)hq * D + dim] = outv;
    } else {
      uint16_t* kc = P.kv + ((size_t)layer * 2 + 0) * kv_layer + ((size_t)b * P.nkv + grp) * head_stride;
      kc[(size_t)pos * D + dim] = f2bf(outv);
    }
  } else {
    const int dim = rr - (G + 1) * D;
    uint16_t* vc = P.kv + ((size_t)layer * 2 + 1) * kv_layer + ((size_t)b * P.nkv + grp) * head_stride;
    vc[(size_t)pos * D + dim] = f2bf(v);
  }
}

template <int BM>
__device__ __forceinline__ void epi_qkv(const DecodeParams& P, const DSmem& S, const Task& t, float r, int st,
                                        float2 cs) {
  const int tid = threadIdx.x;
  const int b = tid % BM;
  if (tid >= (int)t.nrows * BM || b >= P.nb) return;
  // the RoPE partner row (R ^ 1) of the same sequence sits at tid ^ BM
  qkv_out(P, t.layer, (int)t.row0 + tid / BM, b, S.tot[tid] * r, S.tot[tid ^ BM] * r, st, cs);
}

// ---------------------------------------------------------------------------------------
// Split-KV attention chunk for one (sequence, KV head): scores of its G query heads over the
// chunk's keys, per-warp online softmax, merged across warps into one partial (m, l, acc).
// At the current length only nch_eff = ceil(L / min_chunk_keys) (at most nch) chunks hold keys;
// the other chunk tasks only count their arrival.  The last task of the (sequence, KV head)
// to arrive merges the partials into o (FlashDecoding-style online-softmax merge) and
// notifies; with a single chunk in use that chunk writes o directly and nothing is merged.
//
// Keys before the current position were written by earlier steps, so they stream through the
// weight ring like weights: the producer copies the chunk's old K and V rows (kv_stage_keys
// per stage, K rows then V rows) in queue order, ahead of the task's release, and the workers
// read them from shared memory.  Only q and the key/value at the current position (written by
// this step's QKV tasks) are loaded after the release; with QK-norm the task also normalises
// and rotates q and that key (qk_norm_rope).  Each lane holds DL = D/32 dims of
// every head; the kAttnBlock x 4 (key, head) partial dot products of a block are summed
// across lanes with one transposed butterfly (each exchange halves the live values) and
// broadcast back with shuffles.
constexpr int kAttnBlock = 8;  // keys per warp per block
template <int D>
__host__ __device__ constexpr int kv_stage_keys() { return kSlotBytes / (2 * D * 2); }

// How the chunk tasks of a (sequence, KV head) share the work at one step.
enum AttnMode : int {
  AM_SPLIT = 0,     // chunk c takes keys [j0, j1) for all G heads; the last to arrive merges
  AM_HEAD = 1,      // short length: chunk c < G takes query head c over every key, no merge
  AM_INACTIVE = 2,  // sequence outside the active batch: nothing to compute
};

struct AttnGeom {
  int b, g, c, Lk, nch_eff, j0, j1, pos0;
  int mode;  // AttnMode
  int h0;    // first query head of the task within the group (head mode: c)
  int gh;    // query heads the task computes (G, or 1 in head mode)
};

// Chunk of an attention task at step st of the launch: keys [j0, j1) of Lk = pos + 1; pos0 is
// the sequence's position at the launch's first step (rows at or past it are written during
// this launch).  Up to head_keys keys (and with G > 1 query heads per KV head, at least G
// chunks) the group runs in head mode: every key of one query head per chunk, so no partial
// is merged; the chunks c >= G have no work.  Longer lengths split the keys.
__device__ __forceinline__ AttnGeom attn_geom(const DecodeParams& P, const Task& t, int st) {
  AttnGeom a;
  const int G = P.nq / P.nkv;
  a.b = (int)t.row0 / P.nkv;
  a.g = (int)t.row0 % P.nkv;
  a.c = t.aux;
  a.pos0 = P.pos[a.b];
  a.Lk = P.pos[a.b] + st + 1;
  a.h0 = 0;
  a.gh = G;
  if (a.b >= P.nb) {  // sequence not in the active batch: its tasks only count their arrival
    a.mode = AM_INACTIVE;
    a.nch_eff = 0;
    a.j0 = a.j1 = 0;
    return a;
  }
  if (G > 1 && P.nch >= G && a.Lk <= P.head_keys) {
    a.mode = AM_HEAD;
    a.nch_eff = G;
    a.h0 = a.c < G ? a.c : 0;
    a.gh = 1;
    a.j0 = 0;
    a.j1 = a.c < G ? a.Lk : 0;
    return a;
  }
  a.mode = AM_SPLIT;
  a.nch_eff = max(1, min(P.nch, (a.Lk + P.min_chunk_keys - 1) / P.min_chunk_keys));
  const int cl = (a.Lk + a.nch_eff - 1) / a.nch_eff;
  a.j0 = a.c * cl;
  a.j1 = (a.c < a.nch_eff) ? min(a.Lk, a.j0 + cl) : a.j0;
  return a;
}

template <int D>
__device__ __forceinline__ const uint16_t* attn_cache(const DecodeParams& P, const Task& t, const AttnGeom& a,
                                                       int kind) {
  const size_t head_stride = (size_t)P.max_seq * D;
  const size_t kv_layer = (size_t)P.max_batch * P.nkv * head_stride;
  return P.kv + ((size_t)t.layer * 2 + kind) * kv_layer + ((size_t)a.b * P.nkv + a.g) * head_stride;
}

template <int D>
__device__ __forceinline__ void attn_load_key(const uint16_t* kc, const uint16_t* vc, int j, int lane,
                                              uint32_t (&kw)[D / 64], uint32_t (&vw)[D / 64]) {
  if (D == 128) {
    const uint2 a = ldcg_u2(kc + (size_t)j * D + lane * 4);
    const uint2 b = ldcg_u2(vc + (size_t)j * D + lane * 4);
    kw[0] = a.x; kw[(D / 64) - 1] = a.y;
    vw[0] = b.x; vw[(D / 64) - 1] = b.y;
  } else {
    kw[0] = ldcg_u32(kc + (size_t)j * D + lane * 2);
    vw[0] = ldcg_u32(vc + (size_t)j * D + lane * 2);
  }
}

// QK-norm (Mirage article, "Case 4.1: Attention with Query-Key Normalization"): LayerNorm of
// one head held by a warp (lane l holds dims l*DL .. l*DL + DL-1), with this lane's gains g and
// biases bi of the head, then RoPE with this lane's angles cs of the position.  The
// rotate-half partner of dim d < D/2 is d + D/2, held by lane l ^ 16 at the same register
// index.  Warp-uniform.
template <int D>
__device__ __forceinline__ void qk_norm_rope(float (&v)[D / 32], const float (&g)[D / 32], const float (&bi)[D / 32],
                                             const float2 (&cs)[D / 32], float eps, int lane) {
  constexpr int DL = D / 32;
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < DL; ++i) sum += v[i];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float mean = sum * (1.0f / D);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < DL; ++i) {
    v[i] -= mean;
    sq = fmaf(v[i], v[i], sq);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  const float r = 1.0f / sqrtf(sq * (1.0f / D) + eps);
#pragma unroll
  for (int i = 0; i < DL; ++i) v[i] = fmaf(v[i] * r, g[i], bi[i]);
  const bool hi = lane >= 16;
#pragma unroll
  for (int i = 0; i < DL; ++i) {
    const float o = __shfl_xor_sync(0xffffffffu, v[i], 16);
    v[i] = hi ? fmaf(v[i], cs[i].x, o * cs[i].y) : fmaf(v[i], cs[i].x, -(o * cs[i].y));
  }
}

// QK-norm gains and biases of a layer: q gain [nq*D], q bias [nq*D], k gain [nkv*D], k bias [nkv*D].
__device__ __forceinline__ const uint16_t* qk_norm_params(const DecodeParams& P, int layer) {
  return reinterpret_cast<const uint16_t*>(P.arena + P.loff[layer].qkn);
}

// This lane's DL gains (or biases) of head row `head` of a QK-norm parameter array.
template <int D>
__device__ __forceinline__ void qk_param_load(const uint16_t* base, int head, int lane, float (&out)[D / 32]) {
  const uint16_t* p = base + (size_t)head * D + lane * (D / 32);
  if constexpr (D == 128) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    out[0] = __uint_as_float(u.x << 16);
    out[1] = __uint_as_float(u.x & 0xffff0000u);
    out[2] = __uint_as_float(u.y << 16);
    out[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(p));
    out[0] = __uint_as_float(u << 16);
    out[1] = __uint_as_float(u & 0xffff0000u);
  }
}

// Before an attention task's release (its inputs need not exist yet): bring this lane's QK-norm
// gains, biases and RoPE angles into L1, so the norm after the release finds them there.
template <int D>
__device__ __forceinline__ void qk_norm_prefetch(const DecodeParams& P, const Task& t, int st, int lane) {
  const AttnGeom a = attn_geom(P, t, st);
  if (a.c >= a.nch_eff) return;
  const int G = P.nq / P.nkv;
  const uint16_t* nb = qk_norm_params(P, t.layer);
  const int off = lane * (D / 32);
  for (int h = 0; h < G; ++h) {
    prefetch_l1(nb + (size_t)(a.g * G + h) * D + off);
    prefetch_l1(nb + (size_t)(P.nq + a.g * G + h) * D + off);
  }
  prefetch_l1(nb + (size_t)(2 * P.nq + a.g) * D + off);
  prefetch_l1(nb + (size_t)(2 * P.nq + P.nkv + a.g) * D + off);
  prefetch_l1(P.rope + (size_t)(a.Lk - 1) * (D / 2) + (lane & 15) * (D / 32));
}

// Online-softmax update of this warp's (m, l, acc) with one block of up to kAttnBlock keys
// (K and V words kw/vw of this lane; key u counts if bit u of `valid` is set) for the GW
// (1, 2 or 4, a power of two >= G) query heads of the KV head.  The kAttnBlock x GW partial
// dots (slot u * GW + h) are summed across lanes by warp_reduce_rows, which leaves slot r on
// the lanes l with l % (32 / slots) == 0, and are then broadcast to every lane.
template <int D, int GW>
__device__ __forceinline__ void attn_block(const float (&qv)[4][D / 32], const uint32_t (&kw)[kAttnBlock][D / 64],
                                           const uint32_t (&vw)[kAttnBlock][D / 64], uint32_t valid, int G,
                                           float (&m)[4], float (&l)[4], float (&acc)[4][D / 32], int lane) {
  constexpr int DL = D / 32;
  constexpr int W = D / 64;
  constexpr int NS = kAttnBlock * GW;  // slots
  float sc[NS];
#pragma unroll
  for (int u = 0; u < kAttnBlock; ++u) {
    float kf[DL];
#pragma unroll
    for (int w = 0; w < W; ++w) {
      kf[2 * w] = bf16lo(kw[u][w]);
      kf[2 * w + 1] = bf16hi(kw[u][w]);
    }
#pragma unroll
    for (int h = 0; h < GW; ++h) {
      float sv = 0.f;
#pragma unroll
      for (int i = 0; i < DL; ++i) sv = fmaf(qv[h][i], kf[i], sv);
      sc[u * GW + h] = sv;
    }
  }
  // transposed butterfly (each exchange halves the live values), then a plain one: lane l
  // ends with the warp total of slot r = l >> SH (key u = r / GW, head h = r % GW)
  constexpr int LV = ilog2(NS);
  constexpr int SH = 5 - LV;  // log2(lanes per slot)
  constexpr int LG = ilog2(GW);
#pragma unroll
  for (int k = 0; k < LV; ++k) {
    const int off = 16 >> k, half = (NS >> k) >> 1;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? sc[i] : sc[i + half];
      const float keep = upper ? sc[i + half] : sc[i];
      sc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 >> LV; off >= 1; off >>= 1) sc[0] += __shfl_xor_sync(0xffffffffu, sc[0], off);
  // online softmax with one exponential per lane: each lane owns its slot's score
  const int r = lane >> SH, u_me = r >> LG, h_me = r & (GW - 1);
  const bool v_me = ((valid >> u_me) & 1u) && h_me < G;
  const float s_me = v_me ? sc[0] : -INFINITY;
  float mx = s_me;  // block maximum of head h_me: over the key bits of the slot index
#pragma unroll
  for (int k = 0; k < 3; ++k) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1 << (SH + LG + k)));
  float M[GW], alpha[GW];
#pragma unroll
  for (int h = 0; h < GW; ++h) {
    const float bm = __shfl_sync(0xffffffffu, mx, h << SH);  // key 0's lanes hold head h's maximum
    M[h] = fmaxf(m[h], bm);
    alpha[h] = (h < G) ? __expf(m[h] - M[h]) : 0.f;  // 0 on the first block (m = -inf)
  }
  const float p_me = v_me ? __expf(s_me - M[h_me]) : 0.f;
  float ps = p_me;  // block sum of head h_me
#pragma unroll
  for (int k = 0; k < 3; ++k) ps += __shfl_xor_sync(0xffffffffu, ps, 1 << (SH + LG + k));
#pragma unroll
  for (int h = 0; h < GW; ++h) {
    if (h < G) {
      const float bs = __shfl_sync(0xffffffffu, ps, h << SH);
      l[h] = l[h] * alpha[h] + bs;
      m[h] = M[h];
#pragma unroll
      for (int i = 0; i < DL; ++i) acc[h][i] *= alpha[h];
    }
  }
  // P.V: every lane takes each slot's probability from that slot's lanes (the V words of a
  // key outside the block are stale or unset, so they are skipped rather than weighted by 0)
#pragma unroll
  for (int u = 0; u < kAttnBlock; ++u) {
#pragma unroll
    for (int h = 0; h < GW; ++h) {
      const float p = __shfl_sync(0xffffffffu, p_me, (u * GW + h) << SH);
      if (h < G && ((valid >> u) & 1u)) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          acc[h][2 * w] = fmaf(p, bf16lo(vw[u][w]), acc[h][2 * w]);
          acc[h][2 * w + 1] = fmaf(p, bf16hi(vw[u][w]), acc[h][2 * w + 1]);
        }
      }
    }
  }
}

template <int D>
__device__ __forceinline__ void attn_block_g(const float (&qv)[4][D / 32], const uint32_t (&kw)[kAttnBlock][D / 64],
                                             const uint32_t (&vw)[kAttnBlock][D / 64], uint32_t valid, int G,
                                             float (&m)[4], float (&l)[4], float (&acc)[4][D / 32], int lane) {
  if (G == 1) attn_block<D, 1>(qv, kw, vw, valid, G, m, l, acc, lane);
  else if (G == 2) attn_block<D, 2>(qv, kw, vw, valid, G, m, l, acc, lane);
  else attn_block<D, 4>(qv, kw, vw, valid, G, m, l, acc, lane);
}

// Number of ring stages of an attention task: its rows written before the launch,
// [j0, min(j1, pos0)) (the producer runs ahead and must not read rows of this launch).
template <int D>
__device__ __forceinline__ int attn_stage_span(const AttnGeom& a, int* jend) {
  *jend = (a.c < a.nch_eff) ? max(a.j0, min(a.j1, a.pos0)) : a.j0;
  return *jend > a.j0 ? (*jend - a.j0 + kv_stage_keys<D>() - 1) / kv_stage_keys<D>() : 0;
}

// Wide attention (long chunks): WPS warps share a stage.  With WPS = 1 warp w takes ring stages
// w, w + 8, ... whole; with WPS = 2 the warp pair (2p, 2p + 1) takes stages p, p + 4, ..., warp
// 2p + h the stage's key half h (the stage is held half as long, so the ring turns over faster,
// at the price of loading q once per key instead of once per two).  Each warp keeps its own
// online softmax.
// Lane l scores keys l*KPL .. l*KPL + KPL-1 of its half over every dim (reading its K words in
// the rotated order (t + l) mod (D/2), so the 32 lanes hit 32 banks, and the matching q words
// of the scaled q in S.qn), then owns D/32 output dims of P.V, with its half's probabilities
// read back as broadcasts from its row of S.wp.  Stages are taken out of order, so a warp first
// waits until its stage is armed with its launch-wide number (S.armed), then on the stage's
// phase; each warp sharing a stage releases it for 1/WPS of the worker warps.  False if a
// wait ran out (the warp then skips its remaining stages).
constexpr int kWideMinStages = 3;

// One whole stage (or its key half kb .. kb + KPW - 1) of wide attention: kst holds the stage's
// K rows, then its V rows at KPS * D; nk (> 0) keys of this warp.  See attn_wide.
template <int D, int GW, int WPS>
__device__ __forceinline__ void attn_wide_stage(DSmem& S, const uint8_t* kst, int nk, int G, float (&m)[4],
                                                float (&l)[4], float (&acc)[4][D / 32], int lane, int warp) {
  constexpr int KPS = kv_stage_keys<D>();
  constexpr int KPW = KPS / WPS;
  constexpr int W2 = D / 2;
  constexpr int KPL = KPW / 32;
  constexpr int DL = D / 32;
  float* pw = S.wp[warp];  // [GW][KPW]
  const float* qs = S.qn;  // [G][D], scaled
  const int kb = (warp % WPS) * KPW;
  const uint16_t* vst = reinterpret_cast<const uint16_t*>(kst + KPS * D * 2);
  // scores of this lane's keys for every head
  float sc[KPL][GW];
#pragma unroll
  for (int k = 0; k < KPL; ++k)
#pragma unroll
    for (int h = 0; h < GW; ++h) sc[k][h] = 0.f;
  const uint32_t* kwr = reinterpret_cast<const uint32_t*>(kst) + (kb + lane * KPL) * W2;
#pragma unroll 4
  for (int t = 0; t < W2; ++t) {
    const int tr = (t + lane) & (W2 - 1);
    float2 q2[GW];
#pragma unroll
    for (int h = 0; h < GW; ++h)
      q2[h] = (h < G) ? *reinterpret_cast<const float2*>(qs + h * D + 2 * tr) : make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      const uint32_t w = kwr[k * W2 + tr];
      const float k0 = bf16lo(w), k1 = bf16hi(w);
#pragma unroll
      for (int h = 0; h < GW; ++h) sc[k][h] = fmaf(q2[h].y, k1, fmaf(q2[h].x, k0, sc[k][h]));
    }
  }
  // online softmax of each head over the stage's keys
#pragma unroll
  for (int h = 0; h < GW; ++h) {
    if (h >= G) continue;
    float bm = -INFINITY;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      if (lane * KPL + k >= nk) sc[k][h] = -INFINITY;
      bm = fmaxf(bm, sc[k][h]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    const float m_new = fmaxf(m[h], bm);  // finite: the stage holds at least one key
    const float alpha = __expf(m[h] - m_new);
    float psum = 0.f;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      const float p = (lane * KPL + k < nk) ? __expf(sc[k][h] - m_new) : 0.f;
      pw[h * KPW + lane * KPL + k] = p;
      psum += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l[h] = fmaf(l[h], alpha, psum);
    m[h] = m_new;
#pragma unroll
    for (int d = 0; d < DL; ++d) acc[h][d] *= alpha;
  }
  __syncwarp();
  // P.V: lane owns dims lane*DL .. lane*DL + DL-1; keys past nk are skipped (their V bytes are
  // stale, so they are not weighted by 0)
  const uint16_t* vl = vst + (size_t)kb * D + lane * DL;
  const int n4 = nk & ~3;
  for (int k0 = 0; k0 < n4; k0 += 4) {
    float4 p4[GW];
#pragma unroll
    for (int h = 0; h < GW; ++h) p4[h] = *reinterpret_cast<const float4*>(pw + h * KPW + k0);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v[DL];
      if constexpr (DL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(vl + (k0 + e) * D);
        v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
      } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(vl + (k0 + e) * D);
        v[0] = bf16lo(u); v[1] = bf16hi(u);
      }
#pragma unroll
      for (int h = 0; h < GW; ++h) {
        const float p = e == 0 ? p4[h].x : e == 1 ? p4[h].y : e == 2 ? p4[h].z : p4[h].w;
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[h][d] = fmaf(p, v[d], acc[h][d]);
      }
    }
  }
  for (int k = n4; k < nk; ++k) {
    float v[DL];
    if constexpr (DL == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(vl + k * D);
      v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(vl + k * D);
      v[0] = bf16lo(u); v[1] = bf16hi(u);
    }
#pragma unroll
    for (int h = 0; h < GW; ++h) {
      if (h >= G) continue;
      const float p = pw[h * KPW + k];
#pragma unroll
      for (int d = 0; d < DL; ++d) acc[h][d] = fmaf(p, v[d], acc[h][d]);
    }
  }
}

// Tensor-core kernel: the last quarter of a whole-stage chunk's K/V stages are not streamed
// through the ring but loaded into the two activation operand buffers, which attention tasks
// leave idle, by the last warp pair itself (two stages in flight); the other pairs take the
// ring stages.  That is 6 instead of 4 stages in flight per SM.  (A quarter measured best on
// B200 at 16 x 1024 positions: 6.40 ms/step against 6.48 for a third, 6.68 for two fifths,
// 6.43 for a fifth and 6.60 with every stage through the ring.)
static_assert(kTcBopBuf >= kSlotBytes, "a K/V ring stage fits one operand buffer");
template <bool TC>
__device__ __forceinline__ int attn_kv_op_stages(int nst) {
  return (TC && nst >= kWideMinStages) ? nst / 4 : 0;
}

template <int D, int GW, int WPS>
__device__ __forceinline__ bool attn_wide(const DecodeParams& P, DSmem& S, const Pipe& pp, const uint8_t* ring,
                                          const AttnGeom& a, int jend, int nst, int G, float (&m)[4], float (&l)[4],
                                          float (&acc)[4][D / 32], int lane, int warp, uint32_t task_id,
                                          uint32_t& stall_ns, int nb, uint8_t* kvb, uint32_t kvn,
                                          const uint16_t* kc, const uint16_t* vc) {
  constexpr int KPS = kv_stage_keys<D>();  // keys per stage: 64 (D = 128) or 128 (D = 64)
  constexpr int KPW = KPS / WPS;            // keys per warp
  const int kb = (warp % WPS) * KPW;  // this warp's first key in a stage
  const int nr = nst - nb;            // ring stages; operand-buffer stages nr .. nst - 1
  const int np = kAttnWarps / WPS - (nb > 0 ? 1 : 0);  // warp groups on ring stages
  bool ok = true;
  if (warp / WPS < np) {
  for (int i = warp / WPS; i < nr; i += np) {
    int pos = pp.stage + i;
    uint32_t ph = pp.phase;
    while (pos >= pp.nst) {
      pos -= pp.nst;
      ph ^= 1u;
    }
    const uint32_t seq = pp.seq + (uint32_t)i;
    const uint64_t tw = (P.trace && lane == 0 && warp == 0) ? globaltimer_ns() : 0;
    bool got = ok;
    if (got) {  // bounded: the stage armed with this number, then its phase
      uint64_t t0 = 0;
      for (uint32_t n = 1;; ++n) {
        if (ld_acquire_cta_shared(&S.armed[pos]) == seq) break;
        if ((n & 127u) == 0) {
          if (S.abort) {
            got = false;
            break;
          }
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          else if (now - t0 > P.timeout_ns) {
            got = false;
            break;
          }
        }
      }
    }
    got = got && wait_bar(&S.full[pos], ph, P.timeout_ns, &S);
    got = __all_sync(0xffffffffu, got);
    if (tw) stall_ns += (uint32_t)(globaltimer_ns() - tw);
    if (!got) {
      if (ok && lane == 0) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
      ok = false;
      continue;
    }
    const uint8_t* kst = ring + (size_t)pos * kSlotBytes;
    const int nk = min(KPW, min(KPS, jend - (a.j0 + i * KPS)) - kb);  // this warp's keys (none if <= 0)
    if (nk > 0) attn_wide_stage<D, GW, WPS>(S, kst, nk, G, m, l, acc, lane, warp);  // warp-uniform
    __syncwarp();  // every lane's reads of the stage and of pw are done
    if (lane == 0) mbar_arrive_cnt(&S.empty[pos], kWorkerWarps / WPS);
  }
  return ok;
  }
  // the last warp group: operand-buffer stages.  Stage b of the chunk's nb is the CTA's
  // operand-buffer load kvn + b, into buffer (kvn + b) & 1; its first warp's lane 0 issues the
  // loads (the next one into a buffer once both warps released it) and every warp of the
  // group waits for them, so none is left in flight when the task returns.
  const bool lead = (warp % WPS) == 0;  // the group's first warp: its lane 0 issues, it drains
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int b) {
    const uint32_t g = kvn + (uint32_t)b, buf = g & 1u;
    const int jj = a.j0 + (nr + b) * KPS;
    const uint32_t bytes = (uint32_t)min(KPS, jend - jj) * D * 2u;
    uint8_t* dst = kvb + (size_t)buf * kTcBopBuf;
    fence_proxy_async_smem();  // after the generic accesses of the buffer's previous use
    mbar_arrive_expect_tx(&S.kv_full[buf], 2u * bytes);
    bulk_g2s(dst, kc + (size_t)jj * D, bytes, &S.kv_full[buf], pol);
    bulk_g2s(dst + KPS * D * 2, vc + (size_t)jj * D, bytes, &S.kv_full[buf], pol);
  };
  int issued = nb < 2 ? nb : 2;  // loads issued (kept by the lead warp)
  if (lead && lane == 0)
    for (int b = 0; b < issued; ++b) issue(b);
  int done = 0;  // stages whose load this warp saw land
  for (int b = 0; b < nb && ok; ++b) {
    const uint32_t g = kvn + (uint32_t)b, buf = g & 1u;
    const bool got = __all_sync(0xffffffffu, wait_bar(&S.kv_full[buf], (g >> 1) & 1u, P.timeout_ns, &S));
    if (!got) {
      if (lane == 0) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
      ok = false;
      break;
    }
    done = b + 1;
    const int nk = min(KPW, min(KPS, jend - (a.j0 + (nr + b) * KPS)) - kb);
    if (nk > 0) attn_wide_stage<D, GW, WPS>(S, kvb + (size_t)buf * kTcBopBuf, nk, G, m, l, acc, lane, warp);
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.kv_empty[buf]);
    if (lead && b + 2 < nb) {
      // the buffer's next load, once both warps of the group released it (bounded)
      int fok = 1;
      if (lane == 0) {
        fok = wait_bar(&S.kv_empty[buf], (g >> 1) & 1u, P.timeout_ns, &S) ? 1 : 0;
        if (fok) issue(b + 2);
        else raise_error(P, S, DEV_ERR_WAIT_EMPTY, blockIdx.x, task_id);
      }
      if (!__shfl_sync(0xffffffffu, fok, 0)) {
        ok = false;
        break;
      }
      issued = b + 3;
    }
  }
  // after a wait that ran out: wait (bounded) for the loads issued but not seen landing
  if (lead)
    for (int b = done; b < issued; ++b) {
      const uint32_t g = kvn + (uint32_t)b;
      wait_bar(&S.kv_full[g & 1u], (g >> 1) & 1u, P.timeout_ns, nullptr);
    }
  return ok;
}

// wps: warps per stage (1 or 2).  Head mode keeps whole stages per warp (its chunks are few
// and the weight ring is deep enough); split chunks and the tensor-core kernel's 4-stage ring
// turn over faster with warp pairs (measured on B200).
template <int D>
__device__ __forceinline__ bool attn_wide_g(const DecodeParams& P, DSmem& S, const Pipe& pp, const uint8_t* ring,
                                            const AttnGeom& a, int jend, int nst, int G, int wps, float (&m)[4],
                                            float (&l)[4], float (&acc)[4][D / 32], int lane, int warp,
                                            uint32_t task_id, uint32_t& stall_ns, int nb, uint8_t* kvb,
                                            uint32_t kvn, const uint16_t* kc, const uint16_t* vc) {
#define MK_ATTN_WIDE(GW_, WPS_) \
  attn_wide<D, GW_, WPS_>(P, S, pp, ring, a, jend, nst, G, m, l, acc, lane, warp, task_id, stall_ns, nb, kvb, kvn, kc, vc)
  if (wps == 2) {
    if (G == 1) return MK_ATTN_WIDE(1, 2);
    if (G == 2) return MK_ATTN_WIDE(2, 2);
    return MK_ATTN_WIDE(4, 2);
  }
  if (G == 1) return MK_ATTN_WIDE(1, 1);
  if (G == 2) return MK_ATTN_WIDE(2, 1);
  return MK_ATTN_WIDE(4, 1);
#undef MK_ATTN_WIDE
}

// QKN: the model has QK-norm (a separate instantiation, so the plain path keeps its registers).
template <int D, bool TC, bool QKN>
__device__ __forceinline__ bool attention_task(const DecodeParams& P, DSmem& S, Pipe& pp, const uint8_t* ring,
                                               const Task& t, uint32_t task_id, uint32_t& stall_ns, int st,
                                               uint8_t* kvb, uint32_t& kvn) {
  constexpr int DL = D / 32;
  constexpr int W = D / 64;
  constexpr int KPS = kv_stage_keys<D>();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = P.nq / P.nkv;
  const AttnGeom a = attn_geom(P, t, st);
  const int g = a.g, b = a.b, c = a.c, nch_eff = a.nch_eff, pos = a.Lk - 1;
  const int Gt = a.gh, hb = g * G + a.h0;  // the task's query heads: hb .. hb + Gt - 1
  const uint16_t* kc = attn_cache<D>(P, t, a, 0);
  const uint16_t* vc = attn_cache<D>(P, t, a, 1);
  const float* qsrc = P.qbuf + ((size_t)t.layer * P.B + b) * P.nq * D + (size_t)hb * D;
  // partial of (head h, chunk cc) of this sequence at part_base + (h * nch + cc) * (D + 2)
  float* part_base = P.part + ((size_t)t.layer * P.B + b) * P.nq * (size_t)P.nch * (D + 2);
  float* o = P.obuf + ((size_t)t.layer * P.B + b) * P.nq * D + (size_t)hb * D;

  if (c < nch_eff) {  // uniform across the CTA
    float qv[4][DL], m[4], l[4], acc[4][DL];
    const float* qsrc_n = qsrc;  // where this task's q heads are read from
    if (QKN) {
      // QK-norm: q and the key of the current position arrive as raw projections (qbuf, kraw).
      // Warp h < G normalises and rotates q head h into S.qn; in the one chunk holding the
      // current position, the last warp does the same for that key and writes it, in bf16, to
      // its cache row.  After one barrier every warp reads q from S.qn and the key row from the
      // cache like any other row.  The gains and angles were prefetched into L1 before the
      // release.
      const uint16_t* nb = qk_norm_params(P, t.layer);
      const bool key_here = a.j0 <= pos && pos < a.j1;  // uniform across the CTA
      const int head = warp < Gt ? hb + warp : (warp == kAttnWarps - 1 && key_here) ? 2 * P.nq + g : -1;
      if (head >= 0) {  // warp-uniform
        float v[DL], gn[DL], bn[DL];
        float2 cs[DL];
        const float* src = warp < Gt ? qsrc + warp * D : P.kraw + ((size_t)t.layer * P.B + b) * P.nkv * D + (size_t)g * D;
#pragma unroll
        for (int i = 0; i < DL; ++i) {
          v[i] = ldcg_f32(src + lane * DL + i);
          cs[i] = P.rope[(size_t)pos * (D / 2) + (lane & 15) * DL + i];
        }
        qk_param_load<D>(nb, head, lane, gn);
        qk_param_load<D>(nb, warp < Gt ? P.nq + head : head + P.nkv, lane, bn);
        qk_norm_rope<D>(v, gn, bn, cs, P.eps, lane);
        if (warp < Gt) {
#pragma unroll
          for (int i = 0; i < DL; ++i) S.qn[warp * D + lane * DL + i] = v[i];
        } else {
          uint16_t* kdst = const_cast<uint16_t*>(kc) + (size_t)pos * D + lane * DL;
          if constexpr (D == 128)
            *reinterpret_cast<uint2*>(kdst) = make_uint2((uint32_t)f2bf(v[0]) | ((uint32_t)f2bf(v[1]) << 16),
                                                         (uint32_t)f2bf(v[2]) | ((uint32_t)f2bf(v[3]) << 16));
          else
            *reinterpret_cast<uint32_t*>(kdst) = (uint32_t)f2bf(v[0]) | ((uint32_t)f2bf(v[1]) << 16);
        }
      }
      worker_bar();
      qsrc_n = S.qn;
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int i = 0; i < DL; ++i) {
        qv[h][i] = (h < Gt) ? (QKN ? qsrc_n[h * D + lane * DL + i] : ldcg_f32(qsrc + h * D + lane * DL + i)) * P.attn_scale
                           : 0.f;
        acc[h][i] = 0.f;
      }
    }
    uint32_t kw[kAttnBlock][W], vw[kAttnBlock][W];
    // Rows of this chunk written during the launch ("fresh": the current position and, in a
    // multi-step launch, those of its earlier steps) cannot come through the ring.  They take
    // the free slots after the old rows of the last ring stage; each warp fetches up to
    // kFreshPre of its fresh slots together with q (one L2 round trip) and any others when the
    // stage is processed.  Fresh rows that do not fit (no stage, or no free slot) follow in
    // blocks of kAttnBlock keys per warp read from memory.  With whole stages per warp (wide)
    // the fresh rows start at the first warp after those of the stages (an idle warp while
    // the stages take fewer than all warps, else one of the first stages, which are in the ring
    // at the release), and that warp fetches its first kFreshPre of them with q.
    constexpr int kFreshPre = 2;
    const int jf0 = max(a.j0, a.pos0), nf = max(0, a.j1 - jf0);
    int jend;
    const int nst = attn_stage_span<D>(a, &jend);
    const bool wide = nst >= kWideMinStages;  // long chunk: whole stages per warp (attn_wide)
    const int wps = (a.mode == AM_HEAD && !TC) ? 1 : 2;  // wide: warps per stage
    const int nl = (nst > 0) ? (jend - a.j0) - (nst - 1) * KPS : 0;  // old rows in the last stage
    const int n_in = (nst > 0 && !wide) ? min(nf, KPS - nl) : 0;     // fresh rows in its free slots
    const int f_first = ((warp - nl) % kAttnWarps + kAttnWarps) % kAttnWarps;  // this warp's first fresh slot
    // this warp's index in the blocks of fresh rows read from memory
    const int fwarp = wide ? ((warp - wps * nst) % kAttnWarps + kAttnWarps) % kAttnWarps : warp;
    uint32_t kpre[kFreshPre][W], vpre[kFreshPre][W];
#pragma unroll
    for (int j = 0; j < kFreshPre; ++j) {
      if (f_first + kAttnWarps * j < n_in)
        attn_load_key<D>(kc, vc, jf0 + f_first + kAttnWarps * j, lane, kpre[j], vpre[j]);
      else if (wide && fwarp + kAttnWarps * j < nf)
        attn_load_key<D>(kc, vc, jf0 + fwarp + kAttnWarps * j, lane, kpre[j], vpre[j]);
    }
    if (wide) {
      // the scaled q of the group's heads in shared memory, read rotated by every lane (with
      // QK-norm S.qn already holds q, which every warp has first read into its registers)
      if (QKN) worker_bar();
      for (int e = tid; e < Gt * D; e += kWorkerThreads)
        S.qn[e] = (QKN ? S.qn[e] : ldcg_f32(qsrc + e)) * P.attn_scale;
      worker_bar();
      const int nb = attn_kv_op_stages<TC>(nst);  // stages loaded into the operand buffers
      if (!attn_wide_g<D>(P, S, pp, ring, a, jend, nst, Gt, wps, m, l, acc, lane, warp, task_id, stall_ns, nb, kvb,
                          kvn, kc, vc))
        S.cabort = 1u;
      kvn += (uint32_t)nb;
      for (int k = 0; k < nst - nb; ++k) pp.advance();
    }
    // old positions from the ring, kv_stage_keys per stage (K rows at 0, V rows at KPS * D)
    for (int st = 0; st < (wide ? 0 : nst); ++st) {
      const int jj = a.j0 + st * KPS, nk = min(KPS, jend - jj);
      const uint64_t tw = (P.trace && tid == 0) ? globaltimer_ns() : 0;
      if (!wait_bar(&S.full[pp.stage], pp.phase, P.timeout_ns, &S)) {
        raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
        S.cabort = 1u;
      }
      if (P.trace && tid == 0) stall_ns += (uint32_t)(globaltimer_ns() - tw);
      const uint8_t* kst = ring + (size_t)pp.stage * kSlotBytes;
      const uint8_t* vst = kst + KPS * D * 2;
      const bool last = st == nst - 1;
#pragma unroll
      for (int kb = 0; kb < KPS / (kAttnBlock * kAttnWarps); ++kb) {
        uint32_t valid = 0;
#pragma unroll
        for (int u = 0; u < kAttnBlock; ++u) {
          const int idx = kb * kAttnBlock * kAttnWarps + warp + u * kAttnWarps;
          if (idx < nk) {
            valid |= 1u << u;
            if (D == 128) {
              const uint2 kk = *reinterpret_cast<const uint2*>(kst + idx * D * 2 + lane * 8);
              const uint2 vv = *reinterpret_cast<const uint2*>(vst + idx * D * 2 + lane * 8);
              kw[u][0] = kk.x; kw[u][W - 1] = kk.y;
              vw[u][0] = vv.x; vw[u][W - 1] = vv.y;
            } else {
              kw[u][0] = *reinterpret_cast<const uint32_t*>(kst + idx * D * 2 + lane * 4);
              vw[u][0] = *reinterpret_cast<const uint32_t*>(vst + idx * D * 2 + lane * 4);
            }
          } else if (last && idx - nk < n_in) {  // a fresh row in a free slot
            const int f = idx - nk, j = (f - f_first) / kAttnWarps;
            valid |= 1u << u;
            if (j < kFreshPre) {
#pragma unroll
              for (int w = 0; w < W; ++w) {
                kw[u][w] = kpre[j < kFreshPre ? j : 0][w];
                vw[u][w] = vpre[j < kFreshPre ? j : 0][w];
              }
            } else {
              attn_load_key<D>(kc, vc, jf0 + f, lane, kw[u], vw[u]);
            }
          }
        }
        if (valid) attn_block_g<D>(qv, kw, vw, valid, Gt, m, l, acc, lane);
      }
      // release the stage: one arrival per warp once its reads are done
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[pp.stage]);
      pp.advance();
    }
    // fresh rows that found no free slot: blocks read from memory
    for (int fb = n_in; fb < nf; fb += kAttnBlock * kAttnWarps) {
      uint32_t valid = 0;
#pragma unroll
      for (int u = 0; u < kAttnBlock; ++u) {
        const int idx = fb + fwarp + u * kAttnWarps;
        if (idx < nf) {
          valid |= 1u << u;
          if (wide && fb == 0 && u < kFreshPre) {  // fetched with q
#pragma unroll
            for (int w = 0; w < W; ++w) {
              kw[u][w] = kpre[u < kFreshPre ? u : 0][w];
              vw[u][w] = vpre[u < kFreshPre ? u : 0][w];
            }
          } else {
            attn_load_key<D>(kc, vc, jf0 + idx, lane, kw[u], vw[u]);
          }
        }
      }
      if (valid) attn_block_g<D>(qv, kw, vw, valid, Gt, m, l, acc, lane);
    }
    // cross-warp merge of this chunk
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h < Gt && warp < kAttnWarps) {
        if (lane == 0) {
          S.am[warp][h] = m[h];
          S.al[warp][h] = l[h];
        }
#pragma unroll
        for (int i = 0; i < DL; ++i) S.aacc[warp][h][lane * DL + i] = acc[h][i];
      }
    }
    worker_bar();
    if (S.cabort) return false;  // a ring wait ran out (uniform: written before the barrier)
    for (int e = tid; e < Gt * D; e += kWorkerThreads) {
      const int h = e / D, d = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, S.am[w][h]);
      float ls = 0.f, as = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
          const float f = __expf(S.am[w][h] - M);
          ls += f * S.al[w][h];
          as += f * S.aacc[w][h][d];
        }
      }
      if (nch_eff == 1 || a.mode == AM_HEAD) {
        o[(size_t)h * D + d] = as / ls;  // the head's only chunk: final output, nothing to merge
      } else {
        float* pc = part_base + ((size_t)(g * G + h) * P.nch + c) * (D + 2);
        pc[2 + d] = as;
        if (d == 0) {
          pc[0] = M;
          pc[1] = ls;
        }
      }
    }
  }
  worker_bar();
  if (a.mode == AM_HEAD) {
    // No merge: the group's event count (nch per group and step) comes from every head task (1
    // each, once its output is stored) and from chunk G for the chunks without work (nch - G).
    // The arrival counter of split-mode steps advances by nch as if every chunk had arrived (one
    // chunk adds it, before its release, which orders it for later steps).
    if (tid == 0) {
      const int c_cnt = P.nch > G ? G : 0;
      if (c == c_cnt) red_relaxed_gpu_add(P.acnt + ((size_t)t.layer * P.B + b) * P.nkv + g, (uint32_t)P.nch);
      const uint32_t add = c < G ? 1u : (c == G ? (uint32_t)(P.nch - G) : 0u);
      if (add && (int)t.notify[0] != P.drop_event) red_release_gpu_add(&P.ev[t.notify[0]], add);
    }
    (void)task_id;
    return true;
  }
  if (tid == 0) {
    uint32_t* cnt = P.acnt + ((size_t)t.layer * P.B + b) * P.nkv + g;
    const uint32_t old = atom_acq_rel_gpu_add(cnt, 1u);
    S.flag = (old + 1u == (P.epoch + (uint32_t)st) * (uint32_t)P.nch) ? 1u : 0u;
  }
  worker_bar();
  if (S.flag && nch_eff > 1) {
    // Merge in one L2 round trip: every thread issues the partial-accumulator loads of its
    // (up to two) output elements together with the (m, l) loads, then weighs each chunk by
    // exp(m_c - M) itself.  Blocks of 16 chunks (one block up to nch_eff = 16).
    const int e0 = tid, e1 = tid + kWorkerThreads;
    const bool has0 = e0 < G * D, has1 = e1 < G * D;
    const int h0 = e0 / D, d0 = e0 % D, h1 = e1 / D, d1 = e1 % D;
    const float* ph0 = part_base + (size_t)(g * G + (has0 ? h0 : 0)) * P.nch * (D + 2) + 2 + d0;
    const float* ph1 = part_base + (size_t)(g * G + (has1 ? h1 : 0)) * P.nch * (D + 2) + 2 + d1;
    float num0 = 0.f, den0 = 0.f, num1 = 0.f, den1 = 0.f;
    for (int c0 = 0; c0 < nch_eff; c0 += 16) {
      float v0[16], v1[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const bool ok = c0 + k < nch_eff;
        v0[k] = (ok && has0) ? ldcg_f32(ph0 + (size_t)(c0 + k) * (D + 2)) : 0.f;
        v1[k] = (ok && has1) ? ldcg_f32(ph1 + (size_t)(c0 + k) * (D + 2)) : 0.f;
      }
      if (c0 == 0) {
        for (int e = tid; e < G * nch_eff; e += kWorkerThreads) {
          const int h = e / nch_eff, cc = e % nch_eff;
          const float* pc = part_base + ((size_t)(g * G + h) * P.nch + cc) * (D + 2);
          S.mg.mm[e] = ldcg_f32(pc);
          S.mg.ll[e] = ldcg_f32(pc + 1);
        }
        worker_bar();
      }
      const float* mm0 = S.mg.mm + (has0 ? h0 : 0) * nch_eff;
      const float* mm1 = S.mg.mm + (has1 ? h1 : 0) * nch_eff;
      float M0 = -INFINITY, M1 = -INFINITY;
      for (int cc = 0; cc < nch_eff; ++cc) {
        M0 = fmaxf(M0, mm0[cc]);
        M1 = fmaxf(M1, mm1[cc]);
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (c0 + k < nch_eff) {
          const int cc = c0 + k;
          const float w0 = (mm0[cc] == -INFINITY) ? 0.f : __expf(mm0[cc] - M0);
          const float w1 = (mm1[cc] == -INFINITY) ? 0.f : __expf(mm1[cc] - M1);
          num0 = fmaf(w0, v0[k], num0);
          den0 = fmaf(w0, S.mg.ll[(has0 ? h0 : 0) * nch_eff + cc], den0);
          num1 = fmaf(w1, v1[k], num1);
          den1 = fmaf(w1, S.mg.ll[(has1 ? h1 : 0) * nch_eff + cc], den1);
        }
      }
    }
    if (has0) o[(size_t)h0 * D + d0] = num0 / den0;
    if (has1) o[(size_t)h1 * D + d1] = num1 / den1;
    worker_bar();
  }
  // the merge stands for every chunk of the group: nch counts of the event
  if (S.flag && tid == 0 && (int)t.notify[0] != P.drop_event) red_release_gpu_add(&P.ev[t.notify[0]], (uint32_t)P.nch);
  (void)task_id;
  return true;
}

// LM-head epilogue: logits and this task's (max, index) partial; the last LM task picks the token.
__device__ __forceinline__ void argmax_merge(float& v, int& idx, float ov, int oi) {
  if (ov > v || (ov == v && oi < idx)) {
    v = ov;
    idx = oi;
  }
}

__device__ __forceinline__ void block_argmax(DSmem& S, float& v, int& idx) {
  const int tid = threadIdx.x, lane = tid & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1)
    argmax_merge(v, idx, __shfl_xor_sync(0xffffffffu, v, off), __shfl_xor_sync(0xffffffffu, idx, off));
  if (lane == 0) {
    S.lmv[tid >> 5] = v;
    S.lmi[tid >> 5] = idx;
  }
  worker_bar();
  if (tid == 0)
    for (int w = 1; w < kWorkerWarps; ++w) argmax_merge(v, idx, S.lmv[w], S.lmi[w]);
}

// The token pick of step st: greedy tokens to next_tokens[st][b]; then the event the next
// step's embedding waits for.
// The step's tokens are picked.  With run-time claims this also zeroes the claim counters of
// the step two ahead (every SM finished its claims of two steps back: each ends its step with
// a static LM-head task, and this is the step's last LM-head task), published by the release.
__device__ __forceinline__ void announce_tokens(const DecodeParams& P, DSmem& S, int st) {
  worker_bar();
  if (P.dyn) {
    uint32_t* row = P.pcnt + (size_t)((P.epoch + (uint32_t)st + 2u) & 3u) * P.n_pools;
    for (int p = threadIdx.x; p < P.n_pools; p += kWorkerThreads) row[p] = 0u;
    worker_bar();
  }
  if (threadIdx.x == 0) red_release_gpu_add(&P.ev[P.ev_tok], 1u);
}

// Tensor parallel: every rank's best (value, vocab index) of the step, exchanged through the
// ranks' slot arrays; each rank waits (bounded) for all of them and picks the same token.
// False (for every worker alike) if the wait ran out.
__device__ __forceinline__ bool tp_exchange_argmax(const DecodeParams& P, DSmem& S, int b, float& v, int& idx,
                                                   int st) {
  const int tid = threadIdx.x;
  if (tid == 0) {
    const uint64_t w = ((uint64_t)__float_as_uint(v) << 32) | (uint32_t)idx;
    for (int d = 0; d < P.tp_ranks; ++d) P.tp_lmx[d][(size_t)P.tp_rank * P.B + b] = w;
    for (int d = 0; d < P.tp_ranks; ++d) red_release_sys_add(P.tp_ev[d] + P.ev_lmx, 1u);
    // each rank raises the counter once per (step, sequence): sequence b of step e is complete
    // at ((e - 1) * nb + b + 1) * ranks
    const uint32_t target =
        (((P.epoch + (uint32_t)st - 1u) * (uint32_t)P.nb) + (uint32_t)b + 1u) * (uint32_t)P.tp_ranks;
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
      if ((int32_t)(ld_acquire_sys(&P.ev[P.ev_lmx]) - target) >= 0) break;
      if ((n & 63u) == 0) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (S.abort || now - t0 > P.timeout_ns) {
          raise_error(P, S, DEV_ERR_WAIT_EVENT, P.ev_lmx, 0u);
          S.cabort = 1u;
          break;
        }
      }
    }
    if (!S.cabort) {
      v = -INFINITY;
      idx = 0x7fffffff;
      for (int r = 0; r < P.tp_ranks; ++r) {
        const uint64_t w2 = ld_acquire_sys_u64(P.tp_lmx[P.tp_rank] + (size_t)r * P.B + b);
        argmax_merge(v, idx, __uint_as_float((uint32_t)(w2 >> 32)), (int)(uint32_t)w2);
      }
    }
  }
  worker_bar();
  return !S.cabort;
}

template <int BM, bool TP>
__device__ __forceinline__ bool epi_lmhead(const DecodeParams& P, DSmem& S, const Task& t, int K, int st) {
  const int tid = threadIdx.x;
  const int vs = TP ? P.tp_vfull : P.V, vb = TP ? P.tp_vbase : 0;  // logits stride, this shard's first row
  for (int b = 0; b < P.nb; ++b) {
    const float r = norm_factor(S, K, P.eps, b);
    float v = -INFINITY;
    int idx = 0x7fffffff;
    for (int i = tid; i < (int)t.nrows; i += kWorkerThreads) {
      const float lv = S.tot[i * BM + b] * r;
      P.logits[(size_t)b * vs + vb + t.row0 + i] = lv;
      argmax_merge(v, idx, lv, vb + (int)t.row0 + i);
    }
    block_argmax(S, v, idx);
    if (tid == 0) {
      P.lm_val[(size_t)t.index * P.B + b] = v;
      P.lm_idx[(size_t)t.index * P.B + b] = idx;
    }
    worker_bar();  // S.lmv / S.lmi are reused by the next sequence
  }
  if (tid == 0) {
    const uint32_t old = atom_acq_rel_gpu_add(&P.ev[P.ev_lm], 1u);
    S.flag = (old + 1u == (P.epoch + (uint32_t)st) * (uint32_t)P.n_lm) ? 1u : 0u;
  }
  worker_bar();
  if (S.flag) {
    // every step exchanges (tensor parallel), even without next_tokens, so the counters stay in step
    if (P.next_tokens || TP) {
      for (int b = 0; b < P.nb; ++b) {
        float v = -INFINITY;
        int idx = 0x7fffffff;
        for (int i = tid; i < P.n_lm; i += kWorkerThreads)
          argmax_merge(v, idx, ldcg_f32(P.lm_val + (size_t)i * P.B + b), ldcg_i32(P.lm_idx + (size_t)i * P.B + b));
        block_argmax(S, v, idx);
        if (TP && !tp_exchange_argmax(P, S, b, v, idx, st)) return false;
        if (tid == 0 && P.next_tokens) P.next_tokens[(size_t)st * P.B + b] = idx;
        worker_bar();
      }
    }
    announce_tokens(P, S, st);
  }
  return true;
}

// ---------------------------------------------------------------------------------------
// Tensor-core projection task (batch width kTcBatch): D[128 rows x 32] = W_tile . [x_hi | x_lo]^T
// over the task's K units, on tcgen05 with the accumulator in tensor memory.
//
// Operands.  A = a block of kTcRows x kTcUnitK bf16 weights straight from the ring stage (the
// host stores every projection as such blocks, no-swizzle K-major core matrices: 8 rows x 16
// bytes contiguous, 16 core matrices per 8-row group along K).  B = the activations of up to
// 16 sequences times the norm gain, each split into a bf16 high part and a bf16 low part (the
// rounding residual), so the product keeps about 16 mantissa bits of x; columns 0..15 are the
// high parts, 16..31 the low parts.  D[r][b] + D[r][16 + b] is row r of sequence b.
//
// Split K.  An op's blocks (tile, K unit) are spread evenly over the SMs, so a tile's K range
// can be covered by several tasks on several SMs.  Each task writes its partial [128][16] and
// its per-sequence sum of x^2 to its own record; the last task of the tile to arrive (arrival
// counter) sums the tile's records in slot order (deterministic), applies the fused norm
// factor and runs the op's epilogue.  Every task notifies the op's event after it finishes,
// so the event completes only after the last arriver's epilogue.
constexpr uint32_t kTcIdesc = (1u << 4)                       // D: fp32
                              | (1u << 7) | (1u << 10)        // A, B: bf16
                              | ((uint32_t)(kTcN >> 3) << 17)   // N
                              | ((uint32_t)(kTcRows >> 4) << 24);  // M (A and B K-major: bits 15, 16 = 0)


__device__ __forceinline__ void warp_argmax(float& v, int& idx) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1)
    argmax_merge(v, idx, __shfl_xor_sync(0xffffffffu, v, off), __shfl_xor_sync(0xffffffffu, idx, off));
}

// Operands of a tensor-core task's op: x of sequence 0 and the stride to the next, norm gain
// (null = none), K and the op's row count.
struct TcOp {
  const float* xs;
  const uint16_t* gain;
  int K, xstride, rows;
};

__device__ __forceinline__ TcOp tc_op(const DecodeParams& P, const Task& t, const LayerOff& lo) {
  const size_t lay = (size_t)t.layer * P.B;
  TcOp o;
  o.gain = nullptr;
  o.K = o.xstride = P.H;
  switch (t.kind) {
    case TK_QKV:
      o.xs = P.x_in + lay * P.H;
      o.gain = reinterpret_cast<const uint16_t*>(P.arena + lo.attn_norm);
      o.rows = (P.nq + 2 * P.nkv) * P.D;
      break;
    case TK_OPROJ:
      o.xs = P.obuf + lay * P.nq * P.D;
      o.K = o.xstride = P.nq * P.D;
      o.rows = P.H;
      break;
    case TK_GATEUP:
      o.xs = P.x_mid + lay * P.H;
      o.gain = reinterpret_cast<const uint16_t*>(P.arena + lo.mlp_norm);
      o.rows = 2 * P.F;
      break;
    case TK_DOWN:
      o.xs = P.hbuf + lay * P.F;
      o.K = o.xstride = P.F;
      o.rows = P.H;
      break;
    default:  // LM head
      o.xs = P.x_in + (size_t)P.L * P.B * P.H;
      o.gain = reinterpret_cast<const uint16_t*>(P.arena + P.off_fnorm);
      o.rows = P.V;
      break;
  }
  return o;
}

// Stage activation segment sg (kTcSegUnits K units) of task t into operand buffer gseg & 1,
// after the MMAs that last read that buffer are done.  Warp w stages sequences w and w + 8,
// lane j the 8-element K groups j, j + 32; sequences outside the active batch and K past the
// end are zeros.  Every load of the lane is issued before the first is used.  The sums of x^2
// of the task's K range accumulate in S.tss[tsb].  Each warp arrives on bop_full once its
// stores are visible to the tensor cores.  False if the wait ran out (the caller aborts).
__device__ __forceinline__ bool tc_stage(const DecodeParams& P, DSmem& S, uint8_t* bop, const Task& t,
                                         const LayerOff& lo, int sg, uint32_t gseg, int tsb, uint32_t task_id) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const TcOp op = tc_op(P, t, lo);
  const int nK = (op.K + kTcUnitK - 1) / kTcUnitK;
  const int u0 = (int)t.row0 % nK, nu = (int)t.nrows;
  const int su = min(kTcSegUnits, nu - sg * kTcSegUnits);
  const int k0 = (u0 + sg * kTcSegUnits) * kTcUnitK, ngroups = su * (kTcUnitK / 8);
  const uint32_t buf = gseg & 1u, use = gseg >> 1;
  bool ok = wait_bar(&S.bop_free[buf], (use & 1u) ^ 1u, P.timeout_ns, &S);
  if (!ok) {
    raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
    S.cabort = 1u;
  }
  tc_fence_after();
  uint8_t* ob = bop + buf * kTcBopBuf;
  constexpr int kJ = kTcSegUnits * kTcUnitK / 8 / 32;  // K groups per lane
  float4 xv[2][kJ][2];
  uint4 gv[kJ];
#pragma unroll
  for (int i = 0; i < kJ; ++i) {
    const int j = lane + 32 * i, k = k0 + j * 8;
    const bool in = j < ngroups && k < op.K;
    gv[i] = (in && op.gain) ? __ldg(reinterpret_cast<const uint4*>(op.gain + k))
                            : make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);  // bf16 1.0 pairs
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int b = warp + h * kWorkerWarps;
      if (in && b < P.nb) {
        const float* xb = op.xs + (size_t)b * op.xstride + k;
        xv[h][i][0] = ldcg_f4(xb);
        xv[h][i][1] = ldcg_f4(xb + 4);
      } else {
        xv[h][i][0] = xv[h][i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int b = warp + h * kWorkerWarps;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kJ; ++i) {
      const int j = lane + 32 * i;
      if (j >= ngroups) continue;
      const float4 a = xv[h][i][0], c = xv[h][i][1];
      float x[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
      x[0] *= bf16lo(gv[i].x); x[1] *= bf16hi(gv[i].x);
      x[2] *= bf16lo(gv[i].y); x[3] *= bf16hi(gv[i].y);
      x[4] *= bf16lo(gv[i].z); x[5] *= bf16hi(gv[i].z);
      x[6] *= bf16lo(gv[i].w); x[7] *= bf16hi(gv[i].w);
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint16_t h0 = f2bf(x[2 * q]), h1 = f2bf(x[2 * q + 1]);
        const uint16_t l0 = f2bf(x[2 * q] - bf2f(h0)), l1 = f2bf(x[2 * q + 1] - bf2f(h1));
        hw[q] = (uint32_t)h0 | ((uint32_t)h1 << 16);
        lw[q] = (uint32_t)l0 | ((uint32_t)l1 << 16);
      }
      const int hrow = b, lrow = kTcBatch + b;  // operand rows (MMA N index)
      *reinterpret_cast<uint4*>(ob + (hrow >> 3) * kTcBopSbo + j * 128 + (hrow & 7) * 16) =
          make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(ob + (lrow >> 3) * kTcBopSbo + j * 128 + (lrow & 7) * 16) =
          make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) S.tss[tsb][b] = (sg == 0) ? ss : S.tss[tsb][b] + ss;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&S.bop_full[buf]);
  return ok;
}

// MMA issuer (one thread of the tensor-core kernel's issuer warp): walks the queue like the
// workers; for each tensor-core task waits for a free accumulator, then per segment for the
// staged operand, and issues 8 tcgen05.mma per weight block as the block lands.  Each ring
// stage is released by a commit once its MMAs are done, each operand buffer after its
// segment's MMAs, and the accumulator is announced full after the task's last MMA.
// Attention stages of the ring belong to the workers: the cursor only steps over them.
template <int HD>
__device__ __forceinline__ void tc_issuer(const DecodeParams& P, DSmem& S, const uint8_t* ring, const uint8_t* bop,
                                          uint32_t qb, uint32_t qe, uint32_t tmem) {
  Pipe pp{0, 0, kTcStages, 0};
  uint32_t gseg = 0, gtask = 0;
  const uint32_t b_base0 = smem_u32(bop);
  bool ok = true;
  for (int st = 0; st < P.n_steps && ok; ++st)
  for (uint32_t i = qb; i < qe; ++i) {
    const Task t = P.tasks[i];
    if (t.kind == TK_ATTN) {
      int jend;
      const int nst = attn_stage_span<HD>(attn_geom(P, t, st), &jend);
      for (int k = 0; k < nst - attn_kv_op_stages<true>(nst); ++k) pp.advance();  // its ring stages
      continue;
    }
    if (!is_gemv(t.kind)) continue;
    const uint32_t ab = gtask & 1u, av = gtask >> 1;
    if (!wait_bar(&S.acc_free[ab], (av & 1u) ^ 1u, P.timeout_ns, &S)) {
      if (!S.abort) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, i);
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d_tmem = tmem + ab * kTcN;
    const int nu = (int)t.nrows, nseg = (nu + kTcSegUnits - 1) / kTcSegUnits;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const uint32_t buf = gseg & 1u, use = gseg >> 1;
      if (!wait_bar(&S.bop_full[buf], use & 1u, P.timeout_ns, &S)) {
        if (!S.abort) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, i);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t b_base = b_base0 + buf * kTcBopBuf;
      const int su = min(kTcSegUnits, nu - sg * kTcSegUnits);
      for (int u = 0; u < su; ++u) {
        if (!wait_bar(&S.full[pp.stage], pp.phase, P.timeout_ns, &S)) {
          if (!S.abort) raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, i);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(ring + (size_t)pp.stage * kSlotBytes);
#pragma unroll
        for (int s = 0; s < kTcUnitK / 16; ++s) {
          // K step s: core-matrix columns 2s, 2s + 1 (256 bytes) of the block / of unit u
          const uint64_t ad = tc_smem_desc(a_base + s * 256, 128, (kTcUnitK / 8) * 128);
          const uint64_t bd = tc_smem_desc(b_base + u * (kTcUnitK / 8) * 128 + s * 256, 128, kTcBopSbo);
          tc_mma_f16(d_tmem, ad, bd, kTcIdesc, (sg | u | s) != 0 ? 1u : 0u);
        }
        // the stage's release counts one arrival per worker warp (attention stages are released
        // warp by warp): the issuer's commit arrives as all of them once its MMAs are done
#pragma unroll
        for (int k = 0; k < kWorkerWarps; ++k) tc_commit(&S.empty[pp.stage]);
        pp.advance();
      }
      tc_commit(&S.bop_free[buf]);
      ++gseg;
    }
    if (!ok) break;
    tc_commit(&S.acc_full[ab]);
    ++gtask;
  }
  // leave no MMA in flight: tensor memory is freed after this
  tc_commit(&S.mma_done);
  wait_bar(&S.mma_done, 0, P.timeout_ns, nullptr);
}

// Worker side of a tensor-core task after its segments were staged: wait for the accumulator,
// read it back, then the partial record / tile epilogue.  False (for every worker alike) if a
// wait ran out.
__device__ __forceinline__ bool tc_finish(const DecodeParams& P, DSmem& S, const Task& t, const LayerOff& lo,
                                          uint32_t tmem, uint32_t gtask, int tsb, uint32_t task_id, int st) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t lay = (size_t)t.layer * P.B;
  const TcOp op = tc_op(P, t, lo);
  const uint16_t* gain = op.gain;
  const int K = op.K, rows = op.rows;
  const int nK = (K + kTcUnitK - 1) / kTcUnitK;
  const int tile = (int)t.row0 / nK;
  const uint32_t ab = gtask & 1u, av = gtask >> 1;
  if (!wait_bar(&S.acc_full[ab], av & 1u, P.timeout_ns, &S)) {
    raise_error(P, S, DEV_ERR_WAIT_FULL, blockIdx.x, task_id);
    S.cabort = 1u;
  }
  tc_fence_after();
  worker_bar();
  if (S.cabort) return false;

  // 4. partial record: warps 0-3 read their 32 TMEM lanes (= rows), 32 columns each.  A tile
  //    covered by this task alone goes straight to shared memory and its epilogue.
  const bool solo = t.pad0 == 1;
  float* rec = solo ? S.tile : P.tpart + (size_t)t.index * kTcRecFloats;
  if (warp < 4) {
    float d[32];
    tc_ld32(tmem + ab * kTcN + ((uint32_t)(warp * 32) << 16), d);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.acc_free[ab]);  // the issuer may reuse the accumulator
    float4* dst = reinterpret_cast<float4*>(rec + (warp * 32 + lane) * kTcBatch);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_float4(d[4 * q] + d[kTcBatch + 4 * q], d[4 * q + 1] + d[kTcBatch + 4 * q + 1],
                           d[4 * q + 2] + d[kTcBatch + 4 * q + 2], d[4 * q + 3] + d[kTcBatch + 4 * q + 3]);
  }
  if (tid < kTcBatch) rec[kTcRows * kTcBatch + tid] = S.tss[tsb][tid];
  tc_fence_before();
  worker_bar();
  if (!solo) {
    if (tid == 0) {
      const uint32_t old = atom_acq_rel_gpu_add(&P.tcnt[t.pad1], 1u);
      S.flag = (old + 1u == (P.epoch + (uint32_t)st) * (uint32_t)t.pad0) ? 1u : 0u;
    }
    worker_bar();
    if (!S.flag) return true;
    // 5. last arriver: the tile's records summed in slot order, four records per L2 round trip
    const float* rec0 = P.tpart + (size_t)(t.index - t.aux) * kTcRecFloats;
    constexpr int kE = (kTcRecFloats + kWorkerThreads - 1) / kWorkerThreads;
    float v[kE];
#pragma unroll
    for (int i = 0; i < kE; ++i) v[i] = 0.f;
    for (int sl0 = 0; sl0 < (int)t.pad0; sl0 += 4) {
      float r[4][kE];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kE; ++i) {
          const int e = tid + i * kWorkerThreads;
          r[q][i] = (sl0 + q < (int)t.pad0 && e < kTcRecFloats)
                        ? ldcg_f32(rec0 + (size_t)(sl0 + q) * kTcRecFloats + e)
                        : 0.f;
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kE; ++i) v[i] += r[q][i];
    }
#pragma unroll
    for (int i = 0; i < kE; ++i) {
      const int e = tid + i * kWorkerThreads;
      if (e < kTcRecFloats) S.tile[e] = v[i];
    }
    worker_bar();
  }
  const float* ssum = S.tile + kTcRows * kTcBatch;

  // 6. epilogue: thread tid handles (row, sequence) pairs e = tid + i * 256, e = row * 16 + b
  if (t.kind == TK_LMHEAD) {
    for (int e = tid; e < kTcRows * kTcBatch; e += kWorkerThreads) {
      const int row = e / kTcBatch, b = e % kTcBatch, R = tile * kTcRows + row;
      if (b < P.nb && R < rows)
        P.logits[(size_t)b * P.V + R] = S.tile[e] / sqrtf(ssum[b] / (float)K + P.eps);
    }
    // per-sequence argmax over the tile: warp w takes sequences w and w + 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int b = warp + h * kWorkerWarps;
      if (b < P.nb) {
        const float r = 1.0f / sqrtf(ssum[b] / (float)K + P.eps);
        float v = -INFINITY;
        int idx = 0x7fffffff;
        for (int row = lane; row < kTcRows; row += 32) {
          const int R = tile * kTcRows + row;
          if (R < rows) argmax_merge(v, idx, S.tile[row * kTcBatch + b] * r, R);
        }
        warp_argmax(v, idx);
        if (lane == 0) {
          P.lm_val[(size_t)tile * P.B + b] = v;
          P.lm_idx[(size_t)tile * P.B + b] = idx;
        }
      }
    }
    worker_bar();
    if (tid == 0) {
      const uint32_t old = atom_acq_rel_gpu_add(&P.ev[P.ev_lm], 1u);
      S.flag = (old + 1u == (P.epoch + (uint32_t)st) * (uint32_t)P.n_lm) ? 1u : 0u;
    }
    worker_bar();
    if (S.flag) {
      if (P.next_tokens) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int b = warp + h * kWorkerWarps;
          if (b < P.nb) {
            float v = -INFINITY;
            int idx = 0x7fffffff;
            for (int i = lane; i < P.n_lm; i += 32)
              argmax_merge(v, idx, ldcg_f32(P.lm_val + (size_t)i * P.B + b), ldcg_i32(P.lm_idx + (size_t)i * P.B + b));
            warp_argmax(v, idx);
            if (lane == 0) P.next_tokens[(size_t)st * P.B + b] = idx;
          }
        }
      }
      announce_tokens(P, S, st);
    }
    return true;
  }
  for (int e = tid; e < kTcRows * kTcBatch; e += kWorkerThreads) {
    const int row = e / kTcBatch, b = e % kTcBatch, R = tile * kTcRows + row;
    if (b >= P.nb || R >= rows) continue;
    const float r = gain ? 1.0f / sqrtf(ssum[b] / (float)K + P.eps) : 1.f;
    const float v = S.tile[e] * r;
    switch (t.kind) {
      case TK_QKV: qkv_out(P, t.layer, R, b, v, S.tile[e ^ kTcBatch] * r, st, qkv_rope_angle(P, R, b, st)); break;  // partner row R ^ 1
      case TK_OPROJ: {
        const size_t at = (lay + b) * P.H + R;
        P.x_mid[at] = ldcg_f32(P.x_in + at) + v;
        break;
      }
      case TK_GATEUP:
        if ((R & 1) == 0) {
          const float uv = S.tile[e + kTcBatch] * r;
          P.hbuf[(lay + b) * P.F + R / 2] = v / (1.f + expf(-v)) * uv;
        }
        break;
      default: {  // down
        const size_t at = (lay + b) * P.H + R;
        P.x_in[P.B * P.H + at] = ldcg_f32(P.x_mid + at) + v;
        break;
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------------------------------
// QKN: the model has QK-norm (its own instantiations, so the plain kernels keep their registers).
// DYN: run-time claims (projection tasks taken from per-op pools; TK_POOL queue entries).
// TP: tensor-parallel view (batch width 1, static queues): see DecodeParams.
template <int NSEG_H, int RPS_H, int NSEG_F, int RPS_F, int HD, int BM, bool QKN, bool DYN, bool TP>
__device__ __forceinline__ void decode_body(const DecodeParams& P) {
  constexpr bool TC = BM > kMaxDecodeBatch;  // tensor-core projection tiles
  constexpr int BMC = TC ? 1 : BM;            // CUDA-core GEMV batch width (unused when TC)
  constexpr int NST = ring_stages(TC);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* const bop = ring + (size_t)NST * kSlotBytes;  // tensor-core activation operand
  DSmem& S = *reinterpret_cast<DSmem*>(ring + ring_bytes(TC));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t qb = P.qbegin[blockIdx.x], qe = P.qbegin[blockIdx.x + 1];

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kWorkerWarps);  // one release per worker warp (tensor-core: 8 commits)
    }
    mbar_init(&S.mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.bop_full[b], kWorkerWarps);
      mbar_init(&S.bop_free[b], 1);
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_free[b], 4);
      mbar_init(&S.kv_full[b], 1);
      mbar_init(&S.kv_empty[b], 2);
    }
    S.ready = 0;
    for (int s = 0; s < NST; ++s) S.armed[s] = 0xffffffffu;
    S.dq_n = 0;
    S.wdone = 0;
    S.cabort = 0;
    S.abort = 0;
    S.flag = 0;
    fence_mbar_init();
  }
  if (TC && warp == 0) {  // two 32-column fp32 accumulators (128 lanes) for the whole kernel
    tc_alloc(&S.tmem, 2 * kTcN);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = TC ? S.tmem : 0u;

  if (TC && warp == kIssuerWarp) {
    // ------------------------------- MMA issuer ------------------------------
    if (lane == 0) tc_issuer<HD>(P, S, ring, bop, qb, qe, tmem);
    __syncwarp();
    named_bar_sync(2, kWorkerThreads + 32);  // with the workers, before tensor memory is freed
    return;
  }

  if (warp == kProducerWarp) {
    // ------------------------------- producer -------------------------------
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    // L2 lookahead for dependency stalls: a second cursor over this queue's weight stages.
    // While the ring is full and the producer has been blocked for over kStallPrefetchNs (the
    // workers wait for a dependency, so HBM would idle), it prefetches up to l2_ahead stages
    // beyond the ring into L2; a stage it prefetched later loads from L2.  In steady
    // streaming (short blocks) it prefetches nothing, so it never competes with the ring.
    uint32_t la_task = qb, la_row = 0;
    int la_lead = 0;  // stages the lookahead cursor is in front of the next ring stage
    Task la_t = P.tasks[qb < qe ? qb : 0];  // descriptor under the cursor, cached in registers
    auto la_advance = [&](bool prefetch) {  // move the lookahead cursor one stage on
      while (la_task < qe) {
        if (!is_gemv(la_t.kind) || la_row >= la_t.nrows) {
          if (++la_task < qe) la_t = P.tasks[la_task];
          la_row = 0;
          continue;
        }
        const uint32_t rps = TC ? 1u : (la_t.kind == TK_DOWN) ? (uint32_t)RPS_F : (uint32_t)RPS_H;
        if (prefetch) {
          uint64_t off;
          uint32_t rb;
          gemv_source<TC>(P, la_t, &off, &rb);
          const uint32_t nr = min(rps, la_t.nrows - la_row);
          prefetch_l2(P.arena + off + (uint64_t)(la_t.row0 + la_row) * rb, nr * rb);
        }
        la_row += rps;
        return true;
      }
      return false;
    };
    Pipe pp{0, 0, NST, 0};
    int issued = 0;
    bool ok = true;
    // run-time claims: hand task `id` of step st to the scheduler and workers (FIFO entry),
    // after the workers freed its slot (bounded wait)
    uint32_t dq_count = 0;
    auto dyn_push = [&](uint32_t id, int st) -> bool {
      uint64_t t0 = 0;
      for (uint32_t n = 1;; ++n) {
        if (dq_count - ld_acquire_cta_shared(&S.wdone) < (uint32_t)kDynQ) break;
        if ((n & 63u) == 0) {
          if (S.abort) return false;
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          else if (now - t0 > P.timeout_ns) {
            raise_error(P, S, DEV_ERR_WAIT_EMPTY, blockIdx.x, id);
            return false;
          }
        }
      }
      S.dq_id[dq_count % kDynQ] = id;
      S.dq_st[dq_count % kDynQ] = (uint16_t)st;
      st_release_cta_shared(&S.dq_n, ++dq_count);
      return true;
    };
    // a projection task's weight rows through the ring (i: its task index, for the trace)
    auto stream_gemv = [&](const Task& t, uint32_t i) -> bool {
      uint64_t off;
      uint32_t rb;
      gemv_source<TC>(P, t, &off, &rb);
      const int rps = TC ? 1 : (t.kind == TK_DOWN) ? RPS_F : RPS_H;
      const uint8_t* src = P.arena + off + (uint64_t)t.row0 * rb;
      uint64_t blocked = 0, first = 0;
      for (uint32_t r0 = 0; r0 < t.nrows; r0 += (uint32_t)rps) {
        const uint32_t nr = min((uint32_t)rps, t.nrows - r0);
        const uint64_t tw = (P.trace || P.l2_ahead > 0) ? globaltimer_ns() : 0;
        if (P.l2_ahead > 0 && !mbar_test_now(&S.empty[pp.stage], pp.phase ^ 1u)) {
          // blocked: after kStallPrefetchNs, prefetch while still blocked
          uint64_t t0 = tw;
          for (uint32_t n = 1;; ++n) {
            if (mbar_test(&S.empty[pp.stage], pp.phase ^ 1u)) break;
            const uint64_t now = globaltimer_ns();
            if (now - t0 > kStallPrefetchNs && la_lead < P.l2_ahead && la_advance(true)) {
              ++la_lead;
              t0 = now - kStallPrefetchNs + kStallPrefetchGapNs;  // next prefetch after a short gap
            }
            if ((n & 127u) == 0 && (S.abort || now - tw > P.timeout_ns)) break;
          }
        }
        if (!wait_bar(&S.empty[pp.stage], pp.phase ^ 1u, P.timeout_ns, &S)) {
          if (!S.abort) raise_error(P, S, DEV_ERR_WAIT_EMPTY, blockIdx.x, i);
          return false;
        }
        if (P.trace) {
          const uint64_t now = globaltimer_ns();
          blocked += now - tw;
          if (r0 == 0) first = now;
        }
        mbar_arrive_expect_tx(&S.full[pp.stage], nr * rb);
        bulk_g2s(ring + (size_t)pp.stage * kSlotBytes, src + (uint64_t)r0 * rb, nr * rb, &S.full[pp.stage], pol);
        st_release_cta_shared(&S.armed[pp.stage], pp.seq);
        ++issued;
        // the lookahead cursor stays at or in front of the next ring stage
        if (P.l2_ahead > 0) {
          if (la_lead > 0) --la_lead;
          else la_advance(false);
        }
        pp.advance();
      }
      if (P.trace) {
        P.trace[(size_t)i * kTraceWords + 4] = blocked;
        P.trace[(size_t)i * kTraceWords + 5] = first;
      }
      return true;
    };
    // an attention chunk's old K/V rows through the ring, kv_stage_keys<HD>() per stage: K rows,
    // then V rows (i: its task index, for error reports)
    auto stream_attn = [&](const Task& t, uint32_t i, int st) -> bool {
      const AttnGeom a = attn_geom(P, t, st);
      int jend;
      const int nst = attn_stage_span<HD>(a, &jend);
      const uint16_t* kc = attn_cache<HD>(P, t, a, 0);
      const uint16_t* vc = attn_cache<HD>(P, t, a, 1);
      for (int k = 0; k < nst - attn_kv_op_stages<TC>(nst); ++k) {  // the ring's stages of the chunk
        const int jj = a.j0 + k * kv_stage_keys<HD>();
        const uint32_t bytes = (uint32_t)min(kv_stage_keys<HD>(), jend - jj) * HD * 2u;
        if (!wait_bar(&S.empty[pp.stage], pp.phase ^ 1u, P.timeout_ns, &S)) {
          if (!S.abort) raise_error(P, S, DEV_ERR_WAIT_EMPTY, blockIdx.x, i);
          return false;
        }
        uint8_t* dst = ring + (size_t)pp.stage * kSlotBytes;
        mbar_arrive_expect_tx(&S.full[pp.stage], 2u * bytes);
        bulk_g2s(dst, kc + (size_t)jj * HD, bytes, &S.full[pp.stage], pol);
        bulk_g2s(dst + kv_stage_keys<HD>() * HD * 2, vc + (size_t)jj * HD, bytes, &S.full[pp.stage], pol);
        st_release_cta_shared(&S.armed[pp.stage], pp.seq);
        ++issued;
        pp.advance();
      }
      return true;
    };
    for (int st = 0; st < P.n_steps && ok; ++st) {
    if (st > 0) {  // the lookahead restarts with the step's queue
      la_task = qb;
      la_row = 0;
      la_lead = 0;
      la_t = P.tasks[qb < qe ? qb : 0];
    }
    bool gated = false;
    for (uint32_t i = qb; i < qe && ok; ++i) {
      const Task t = P.tasks[i];
      if constexpr (DYN) {
        if (t.kind == TK_POOL) {
          // this step's claim counters were zeroed by the token pick of the step two back
          if (!gated && st >= 2) {
            const uint32_t target = P.epoch + (uint32_t)st - 2u;
            uint64_t t0 = 0;
            for (uint32_t n = 1;; ++n) {
              if ((int32_t)(ld_acquire_gpu(&P.ev[P.ev_tok]) - target) >= 0) break;
              if ((n & 63u) == 0) {
                if (S.abort || *(volatile uint32_t*)&P.err[ERR_ABORT]) {
                  S.abort = 1u;
                  ok = false;
                  break;
                }
                const uint64_t now = globaltimer_ns();
                if (t0 == 0) t0 = now;
                else if (now - t0 > P.timeout_ns) {
                  raise_error(P, S, DEV_ERR_WAIT_EVENT, P.ev_tok, i);
                  ok = false;
                  break;
                }
              }
            }
            gated = true;
            if (!ok) break;
          }
          // claim until the pool is empty; the next claim is in flight while a task streams.
          // Paced (dyn == 2): a claim waits until the workers have finished every task but the
          // last one handed to them, so an SM holds at most one unstarted task.
          const uint2 pl = P.pools[t.index];
          uint32_t* ctr = P.pcnt + (size_t)((P.epoch + (uint32_t)st) & 3u) * P.n_pools + t.index;
          auto paced = [&]() -> bool {
            if (P.dyn != 2 || dq_count == 0) return true;
            uint64_t t0 = 0;
            for (uint32_t n = 1;; ++n) {
              if (ld_acquire_cta_shared(&S.wdone) + 1u >= dq_count) return true;
              if ((n & 63u) == 0) {
                if (S.abort) return false;
                const uint64_t now = globaltimer_ns();
                if (t0 == 0) t0 = now;
                else if (now - t0 > P.timeout_ns) {
                  raise_error(P, S, DEV_ERR_WAIT_EMPTY, blockIdx.x, i);
                  return false;
                }
              }
            }
          };
          if (!paced()) {
            ok = false;
            break;
          }
          uint32_t c = atomicAdd(ctr, 1u);
          while (ok && c < pl.y) {
            const uint32_t id = pl.x + c;
            if (!dyn_push(id, st)) {
              ok = false;
              break;
            }
            uint32_t cn = 0xffffffffu;
            if (P.dyn != 2) cn = atomicAdd(ctr, 1u);
            {
              const Task tc2 = P.tasks[id];  // a projection tile, or (priority claims) an attention chunk
              ok = tc2.kind == TK_ATTN ? stream_attn(tc2, id, st) : stream_gemv(tc2, id);
            }
            if (ok && P.dyn == 2) {
              ok = paced();
              if (ok) cn = atomicAdd(ctr, 1u);
            }
            c = cn;
          }
          continue;
        }
        if (!dyn_push(i, st)) {
          ok = false;
          break;
        }
      }
      if (t.kind == TK_ATTN) {
        ok = stream_attn(t, i, st);
        continue;
      }
      if (!is_gemv(t.kind)) continue;
      ok = stream_gemv(t, i);
    }
    }
    if (DYN && ok) dyn_push(kDynEnd, 0);
    // leave no copy in flight: wait (bounded) for the last issued stages to land
    for (int k = 1; k <= (issued < NST ? issued : NST); ++k) {
      int s = pp.stage - k;
      uint32_t ph = pp.phase;
      if (s < 0) {
        s += NST;
        ph ^= 1u;
      }
      wait_bar(&S.full[s], ph, P.timeout_ns, nullptr);
    }
    return;
  }

  if (warp == kSchedWarp) {
    // ------------------------------- scheduler ------------------------------
    if (lane != 0) return;
    const uint32_t nq = qe - qb;
    // static queues: entry r is task qb + r % nq of step r / nq; run-time claims: the
    // producer's FIFO entry r (bounded wait for it), up to the end marker
    const uint32_t nr = DYN ? 0xffffffffu : nq * (uint32_t)P.n_steps;
    for (uint32_t r = 0; r < nr; ++r) {
      int st;
      uint32_t i;
      if constexpr (DYN) {
        uint64_t t0 = 0;
        for (uint32_t n = 1;; ++n) {
          if (ld_acquire_cta_shared(&S.dq_n) > r) break;
          if ((n & 63u) == 0) {
            if (S.abort || *(volatile uint32_t*)&P.err[ERR_ABORT]) {
              S.abort = 1u;
              return;
            }
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > P.timeout_ns) {
              raise_error(P, S, DEV_ERR_WAIT_READY, blockIdx.x, r);
              return;
            }
          }
        }
        i = S.dq_id[r % kDynQ];
        if (i == kDynEnd) return;
        st = S.dq_st[r % kDynQ];
      } else {
        st = (int)(r / nq);
        i = qb + r % nq;
      }
      const Task t = P.tasks[i];
      // a later step's embedding also waits for the previous step's token pick
      const int n_wait = t.n_wait + ((t.kind == TK_EMBED && st > 0) ? 1 : 0);
      for (int w = 0; w < n_wait; ++w) {
        const bool tok = w == t.n_wait;
        const uint32_t e = tok ? P.ev_tok : t.wait[w];
        const uint32_t target = tok ? P.epoch + (uint32_t)st - 1u : (P.epoch + (uint32_t)st) * P.ev_count[e];
        uint64_t t0 = 0;
        for (uint32_t n = 1;; ++n) {
          if ((int32_t)((TP ? ld_acquire_sys(&P.ev[e]) : ld_acquire_gpu(&P.ev[e])) - target) >= 0) break;
          if ((n & 63u) == 0) {
            if (S.abort || *(volatile uint32_t*)&P.err[ERR_ABORT]) {
              S.abort = 1u;
              return;
            }
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > P.timeout_ns) {
              raise_error(P, S, DEV_ERR_WAIT_EVENT, e, i);
              return;
            }
          }
        }
      }
      st_release_cta_shared(&S.ready, r + 1u);
    }
    return;
  }

  // --------------------------------- workers ---------------------------------
  Pipe pp{0, 0, NST, 0};
  // tensor-core pipeline (workers): operand segments staged and tasks finished so far, and
  // whether the next task's first segment was staged ahead
  uint32_t gseg = 0, gtask = 0;
  bool staged_ahead = false;
  uint32_t kvn = 0;  // K/V stages loaded into the operand buffers so far (tensor-core attention)
  // batch width 1: the next task's descriptor is loaded during the current task, so only the
  // activation loads remain after its release; wider kernels load it at the top of its own
  // iteration instead, which keeps 10 registers free across the GEMV
  constexpr bool kHoist = (BM == 1) && !DYN;
  Task t_next = P.tasks[qb < qe ? qb : 0];
  // the queue once per step of the launch: k counts released tasks over all steps (run-time
  // claims: the producer's FIFO entries, up to the end marker)
  const uint32_t nq = qe - qb, nk = DYN ? 0xffffffffu : nq * (uint32_t)P.n_steps;
  for (uint32_t k = 0; k < nk; ++k) {
    int st;
    uint32_t i;
    if constexpr (DYN) {
      // the producer's entry k (bounded, abort-aware, then uniform decision)
      uint64_t t0 = 0;
      for (uint32_t n = 1;; ++n) {
        if (ld_acquire_cta_shared(&S.dq_n) > k) break;
        if ((n & 63u) == 0) {
          if (S.abort) {
            S.cabort = 1u;
            break;
          }
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          else if (now - t0 > P.timeout_ns + 1000000000ull) {  // the producer reports first
            raise_error(P, S, DEV_ERR_WAIT_READY, blockIdx.x, k);
            S.cabort = 1u;
            break;
          }
        }
      }
      worker_bar();
      if (S.cabort) break;
      i = S.dq_id[k % kDynQ];
      if (i == kDynEnd) break;
      st = S.dq_st[k % kDynQ];
    } else {
      st = (int)(k / nq);
      i = qb + k % nq;
    }
    const Task t = kHoist ? t_next : P.tasks[i];
    const LayerOff lo = P.loff[t.layer < P.L ? t.layer : 0];
    if (kHoist && k + 1 < nk) t_next = P.tasks[qb + (k + 1) % nq];
    const uint64_t t_wait = (P.trace && tid == 0) ? globaltimer_ns() : 0;
    uint32_t stall = 0;
    if (QKN && t.kind == TK_ATTN) qk_norm_prefetch<HD>(P, t, st, lane);
    // wait for the scheduler to release task i (bounded, abort-aware, then uniform decision)
    {
      uint64_t t0 = 0;
      for (uint32_t n = 1;; ++n) {
        if (ld_acquire_cta_shared(&S.ready) > k) break;
        if ((n & 63u) == 0) {
          if (S.abort) {
            S.cabort = 1u;
            break;
          }
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          else if (now - t0 > P.timeout_ns + 1000000000ull) {  // the scheduler reports first
            raise_error(P, S, DEV_ERR_WAIT_READY, blockIdx.x, i);
            S.cabort = 1u;
            break;
          }
        }
      }
      worker_bar();
      if (S.cabort) break;
    }
    const uint64_t t_ready = (P.trace && tid == 0) ? globaltimer_ns() : 0;
    bool notify = true;
    if (TC && is_gemv(t.kind)) {
      const int nu = (int)t.nrows, nseg = (nu + kTcSegUnits - 1) / kTcSegUnits;
      const int tsb = (int)(gtask & 1u);
      bool ok = true;
      for (int sg = staged_ahead ? 1 : 0; sg < nseg; ++sg) ok &= tc_stage(P, S, bop, t, lo, sg, gseg++, tsb, i);
      staged_ahead = false;
      // the next task of the same op has this task's inputs: stage its first segment now, so
      // the tensor cores go on with it while this task is read back and finished
      const Task tn = P.tasks[i + 1 < qe ? i + 1 : i];
      if (ok && i + 1 < qe && tn.kind == t.kind && tn.layer == t.layer) {
        uint64_t t0 = 0;
        for (uint32_t n = 1;; ++n) {  // its release (immediate: same events as this task)
          if (ld_acquire_cta_shared(&S.ready) > k + 1) break;
          if ((n & 63u) == 0) {
            if (S.abort) {
              ok = false;
              break;
            }
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > P.timeout_ns + 1000000000ull) {
              raise_error(P, S, DEV_ERR_WAIT_READY, blockIdx.x, i + 1);
              ok = false;
              break;
            }
          }
        }
        if (ok) {
          ok = tc_stage(P, S, bop, tn, lo, 0, gseg++, (int)((gtask + 1) & 1u), i + 1);
          staged_ahead = true;
        }
      }
      if (!ok) S.cabort = 1u;
      for (int u = 0; u < nu; ++u) pp.advance();  // the task's weight blocks go to the issuer
      if (!tc_finish(P, S, t, lo, tmem, gtask, tsb, i, st)) goto out;
      ++gtask;
      if (t.kind == TK_LMHEAD) notify = false;
    } else if (is_gemv(t.kind)) {
      // operands of the task's GEMV: x source of sequence 0 and the stride to the next, norm
      // gain (null = no norm) and K
      const float* xs;
      const uint16_t* gain = nullptr;
      int K = P.H, xstride = P.H;
      const size_t lay = (size_t)t.layer * P.B;
      // tensor parallel: the residual stream is the last materialised copy plus every rank's
      // partial rows of the projection that followed it
      XAdd xa{nullptr, 0, nullptr, 0, (size_t)P.B * P.H, nullptr, 0, 0};
      auto recv_of = [&](float* const* bufs, int layer) {
        return bufs[P.tp_rank] + (size_t)layer * P.tp_ranks * P.B * P.H;
      };
      switch (t.kind) {
        case TK_QKV:
          xs = P.x_in + lay * P.H;
          gain = reinterpret_cast<const uint16_t*>(P.arena + lo.attn_norm);
          if (TP && t.layer > 0) {  // x_in[l] = x_mid[l-1] + the ranks' down rows of layer l-1
            xs = P.x_mid + (lay - P.B) * P.H;
            xa.add = recv_of(P.tp_recv_d, t.layer - 1);
            xa.n = P.tp_ranks;
          }
          break;
        case TK_OPROJ:
          xs = P.obuf + lay * P.nq * P.D;
          K = xstride = P.nq * P.D;
          break;
        case TK_GATEUP:
          xs = P.x_mid + lay * P.H;
          gain = reinterpret_cast<const uint16_t*>(P.arena + lo.mlp_norm);
          if (TP) {  // x_mid[l] = x_in[l] + the ranks' O rows, x_in[l] formed as in QKV; written here
            if (t.layer > 0) {
              xs = P.x_mid + (lay - P.B) * P.H;
              xa.add = recv_of(P.tp_recv_d, t.layer - 1);
              xa.n = P.tp_ranks;
            } else {
              xs = P.x_in;  // the embedding
            }
            xa.add2 = recv_of(P.tp_recv_o, t.layer);
            xa.n2 = P.tp_ranks;
            xa.mat = P.x_mid + lay * P.H;
            xa.mlo = (int)t.index;
            xa.mhi = (int)t.pad1;
          }
          break;
        case TK_DOWN: {
          const int k0 = (int)t.aux * P.kdc;  // K chunk of the down projection
          xs = P.hbuf + lay * P.F + k0;
          xstride = P.F;
          K = min(P.kdc, P.F - k0);
          break;
        }
        default:  // LM head
          xs = P.x_in + (size_t)P.L * P.B * P.H;
          gain = reinterpret_cast<const uint16_t*>(P.arena + P.off_fnorm);
          if (TP) {
            xs = P.x_mid + (size_t)(P.L - 1) * P.B * P.H;
            xa.add = recv_of(P.tp_recv_d, P.L - 1);
            xa.n = P.tp_ranks;
          }
          break;
      }
      uint32_t rb;
      {
        uint64_t off_unused;
        gemv_source<false>(P, t, &off_unused, &rb);
      }
      // this thread's (row, sequence) in the epilogues, and the epilogue's other operand, loaded
      // now so that its round trip overlaps the activation loads and the GEMV instead of
      // following them: the residual (O projection, first down chunk), this thread's own sum of
      // the earlier down chunks, or the RoPE angle of its QKV row
      const int eb = tid % BMC, er = tid / BMC;
      const bool mine = er < (int)t.nrows && eb < P.nb;
      float2 e_op = make_float2(1.f, 0.f);  // QKV: (cos, sin); O, down: (residual, -)
      if (mine) {
        const size_t at = (lay + eb) * P.H + t.row0 + er;
        if (t.kind == TK_QKV) e_op = qkv_rope_angle(P, (int)t.row0 + er, eb, st);
        else if (!TP && t.kind == TK_OPROJ) e_op.x = ldcg_f32(P.x_in + at);
        else if (!TP && t.kind == TK_DOWN) e_op.x = (t.aux == 0) ? ldcg_f32(P.x_mid + at) : P.x_in[P.B * P.H + at];
      }
      const bool ok = (t.kind == TK_DOWN)
                          ? gemv_tile<NSEG_F, RPS_F, BMC>(P, S, pp, ring, xs, xstride, P.nb, gain, K, (int)t.nrows, rb,
                                                         i, stall)
                          : gemv_tile<NSEG_H, RPS_H, BMC, TP>(P, S, pp, ring, xs, xstride, P.nb, gain, K, (int)t.nrows,
                                                             rb, i, stall, xa);
      if (!ok) goto out;
      const float r = gain ? norm_factor(S, K, P.eps, eb) : 1.f;
      switch (t.kind) {
        case TK_QKV: epi_qkv<BMC>(P, S, t, r, st, e_op); break;
        case TK_OPROJ:
          if (mine) {
            if constexpr (TP) {  // this rank's partial rows to every rank's receive buffer
              const size_t at = (((size_t)t.layer * P.tp_ranks + P.tp_rank) * P.B + eb) * P.H + t.row0 + er;
              for (int d = 0; d < P.tp_ranks; ++d) P.tp_recv_o[d][at] = S.tot[tid];
            } else {
              P.x_mid[(lay + eb) * P.H + t.row0 + er] = e_op.x + S.tot[tid];
            }
          }
          break;
        case TK_GATEUP:
          if (mine && (er & 1) == 0) {
            const float gv = S.tot[tid] * r, uv = S.tot[tid + BMC] * r;
            const float sg = gv / (1.f + expf(-gv));
            P.hbuf[(lay + eb) * P.F + (t.row0 + er) / 2] = sg * uv;
          }
          break;
        case TK_DOWN:
          if (TP && mine) {
            const size_t at = (((size_t)t.layer * P.tp_ranks + P.tp_rank) * P.B + eb) * P.H + t.row0 + er;
            for (int d = 0; d < P.tp_ranks; ++d) P.tp_recv_d[d][at] = S.tot[tid];
          } else if (mine) {
            // K chunk 0 starts from the residual; later chunks of the same rows ran earlier
            // in this queue, on this thread, and add to what it stored (both in e_op.x)
            P.x_in[P.B * P.H + (lay + eb) * P.H + t.row0 + er] = e_op.x + S.tot[tid];
          }
          break;
        default:
          notify = false;
          if (!epi_lmhead<BMC, TP>(P, S, t, K, st)) goto out;
          break;
      }
    } else if (t.kind == TK_EMBED) {
      for (int b = 0; b < P.nb; ++b) {
        // step 0: the caller's tokens; later steps: the previous step's greedy pick
        int tok = (st == 0) ? ldcg_i32(P.tokens + b) : ldcg_i32(P.next_tokens + (size_t)(st - 1) * P.B + b);
        if (tok < 0 || tok >= (TP ? P.tp_vfull : P.V)) {  // never read outside the table: record, use row 0
          if (tid == 0 && t.row0 == 0) atomicCAS(&P.err[ERR_CODE], 0u, (uint32_t)DEV_ERR_BAD_TOKEN);
          tok = 0;
        }
        const uint16_t* e = reinterpret_cast<const uint16_t*>(P.arena + P.off_embed) + (size_t)tok * P.H;
        for (uint32_t r = tid; r < t.nrows; r += kWorkerThreads)
          P.x_in[(size_t)b * P.H + t.row0 + r] = __uint_as_float((uint32_t)e[t.row0 + r] << 16);
      }
    } else if (t.kind == TK_ATTN) {
      notify = false;  // the last chunk to arrive notifies
      if (!attention_task<HD, TC, QKN>(P, S, pp, ring, t, i, stall, st, bop, kvn)) goto out;
    }
    if (P.trace && tid == 0) {
      uint64_t* rec = P.trace + (size_t)i * kTraceWords;
      rec[0] = t_wait;
      rec[1] = t_ready;
      rec[2] = globaltimer_ns();
      rec[3] = (uint64_t)stall | ((uint64_t)blockIdx.x << 32);
    }
    if (notify) {
      worker_bar();
      if (tid == 0) {
        for (int k = 0; k < t.n_notify; ++k) {
          if ((int)t.notify[k] == P.drop_event) continue;
          if (TP && (t.pad0 & 1u)) {  // remote-signal edge: the event on every rank
            for (int d = 0; d < P.tp_ranks; ++d) red_release_sys_add(P.tp_ev[d] + t.notify[k], 1u);
          } else {
            red_release_gpu_add(&P.ev[t.notify[k]], 1u);
          }
        }
      }
    }
    if constexpr (DYN) {  // every worker read FIFO entry k: its slot can be reused
      worker_bar();
      if (tid == 0) st_release_cta_shared(&S.wdone, k + 1u);
    }
  }
out:
  if (TC) {  // every worker thread and the issuer warp (which drained its MMAs) meet here
    tc_fence_before();
    named_bar_sync(2, kWorkerThreads + 32);
    tc_fence_after();
    if (warp == 0) tc_dealloc(tmem, 2 * kTcN);
  }
}

template <int NSEG_H, int RPS_H, int NSEG_F, int RPS_F, int HD, int BM, bool QKN, bool DYN>
__global__ void __launch_bounds__(BM > kMaxDecodeBatch ? kTcBlockThreads : kBlockThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams P) {
  decode_body<NSEG_H, RPS_H, NSEG_F, RPS_F, HD, BM, QKN, DYN, false>(P);
}

// Several tensor-parallel ranks in one launch on one GPU: CTA b runs rank b / sms_per_rank's
// queue with that rank's view.  On separate GPUs each rank would launch decode_body with its
// own view, its peers' buffers reached through peer mappings.
template <int NSEG_H, int RPS_H, int NSEG_F, int RPS_F, int HD>
__global__ void __launch_bounds__(kBlockThreads, 1) decode_kernel_tp(const __grid_constant__ DecodeParamsTP T) {
  decode_body<NSEG_H, RPS_H, NSEG_F, RPS_F, HD, 1, false, false, true>(T.r[blockIdx.x / T.sms_per_rank]);
}

// ---------------------------------------------------------------------------------------
// Instantiations: (segments, rows per stage) for K = hidden and K = ffn.
// One instantiation per weight-row shape class: (segments, rows per ring stage) of the
// K = hidden and K = ffn GEMVs, computed from representative sizes.
__host__ __device__ constexpr int seg_count(int K) { return (K + kSegElems - 1) / kSegElems; }
__host__ __device__ constexpr int pow2_floor_c(int x) { return x < 2 ? 1 : 2 * pow2_floor_c(x / 2); }
__host__ __device__ constexpr int stage_rows(int K) {
  return pow2_floor_c((kSlotBytes / (2 * K)) < kRpsMax ? (kSlotBytes / (2 * K)) : kRpsMax);
}
// Batch width 1 streams W_down whole (K = ffn); batch width 4 streams it in K chunks of
// kDownChunk columns, so the K = ffn class is the chunk's.
__host__ __device__ constexpr int down_k(int F, int BM) { return BM == 1 ? F : (F < kDownChunk ? F : kDownChunk); }
#define MK_VARIANT(H, F, D, BM, QK, DY) \
  {seg_count(H), stage_rows(H), seg_count(down_k(F, BM)), stage_rows(down_k(F, BM)), D, BM, QK, DY, 0}
#define MK_KERNEL(H, F, D, BM, QK, DY)                                                                           \
  (const void*)decode_kernel<seg_count(H), stage_rows(H), seg_count(down_k(F, BM)), stage_rows(down_k(F, BM)), D, \
                             BM, QK, DY>
// tensor-parallel instantiations: F is one rank's share of the ffn
#define MK_VARIANT_TP(H, F, D) {seg_count(H), stage_rows(H), seg_count(F), stage_rows(F), D, 1, 0, 0, 1}
#define MK_KERNEL_TP(H, F, D) \
  (const void*)decode_kernel_tp<seg_count(H), stage_rows(H), seg_count(F), stage_rows(F), D>
static const Variant kVariants[] = {
    MK_VARIANT(4096, 14336, 128, 1, 0, 0),  // Llama-3-8B shape
    MK_VARIANT(4096, 11008, 128, 1, 0, 0),  // Chameleon-7B shape
    MK_VARIANT(256, 768, 64, 1, 0, 0),      // tiny decoder
    MK_VARIANT(4096, 4096, 128, 1, 0, 0),
    MK_VARIANT(2048, 4096, 128, 1, 0, 0),
    MK_VARIANT(256, 256, 64, 1, 0, 0),
    MK_VARIANT(4096, 4096, 128, 4, 0, 0),   // hidden 4096, any ffn >= 4096 (Llama-3-8B, Chameleon-7B), 2..4 sequences
    MK_VARIANT(256, 768, 64, 4, 0, 0),      // tiny decoder, 2..4 sequences
    MK_VARIANT(2048, 4096, 128, 4, 0, 0),
    MK_VARIANT(256, 256, 64, 4, 0, 0),
    {0, 1, 0, 1, 128, kTcBatch, 0, 0, 0},   // tensor-core projection tiles, 5..16 sequences, any hidden / ffn
    {0, 1, 0, 1, 64, kTcBatch, 0, 0, 0},
    // QK-norm models: Chameleon-7B shape and the tiny decoder, every batch width
    MK_VARIANT(4096, 11008, 128, 1, 1, 0),
    MK_VARIANT(256, 768, 64, 1, 1, 0),
    MK_VARIANT(4096, 4096, 128, 4, 1, 0),
    MK_VARIANT(256, 768, 64, 4, 1, 0),
    {0, 1, 0, 1, 128, kTcBatch, 1, 0, 0},
    {0, 1, 0, 1, 64, kTcBatch, 1, 0, 0},
    // run-time claims (scheduling variant): batch 1, Llama-3-8B shape and the tiny decoder
    MK_VARIANT(4096, 14336, 128, 1, 0, 1),
    MK_VARIANT(256, 768, 64, 1, 0, 1),
    // tensor parallel, batch 1: the tiny decoder over 2 ranks, the Llama-3-8B shape over 2 and 4
    MK_VARIANT_TP(256, 384, 64),
    MK_VARIANT_TP(4096, 7168, 128),
    MK_VARIANT_TP(4096, 3584, 128),
};
static const void* kFns[] = {
    MK_KERNEL(4096, 14336, 128, 1, false, false), MK_KERNEL(4096, 11008, 128, 1, false, false), MK_KERNEL(256, 768, 64, 1, false, false),
    MK_KERNEL(4096, 4096, 128, 1, false, false),  MK_KERNEL(2048, 4096, 128, 1, false, false),  MK_KERNEL(256, 256, 64, 1, false, false),
    MK_KERNEL(4096, 4096, 128, 4, false, false),  MK_KERNEL(256, 768, 64, 4, false, false),     MK_KERNEL(2048, 4096, 128, 4, false, false),
    MK_KERNEL(256, 256, 64, 4, false, false),
    (const void*)decode_kernel<1, 1, 1, 1, 128, kTcBatch, false, false>,
    (const void*)decode_kernel<1, 1, 1, 1, 64, kTcBatch, false, false>,
    MK_KERNEL(4096, 11008, 128, 1, true, false),  MK_KERNEL(256, 768, 64, 1, true, false),
    MK_KERNEL(4096, 4096, 128, 4, true, false),   MK_KERNEL(256, 768, 64, 4, true, false),
    (const void*)decode_kernel<1, 1, 1, 1, 128, kTcBatch, true, false>,
    (const void*)decode_kernel<1, 1, 1, 1, 64, kTcBatch, true, false>,
    MK_KERNEL(4096, 14336, 128, 1, false, true), MK_KERNEL(256, 768, 64, 1, false, true),
    MK_KERNEL_TP(256, 384, 64), MK_KERNEL_TP(4096, 7168, 128), MK_KERNEL_TP(4096, 3584, 128),
};
static_assert(sizeof(kVariants) / sizeof(kVariants[0]) == sizeof(kFns) / sizeof(kFns[0]), "variant table");

int find_decode_variant(int nseg_h, int rps_h, int nseg_f, int rps_f, int head_dim, int bm, int qkn, int dyn, int tp) {
  for (int i = 0; i < (int)(sizeof(kVariants) / sizeof(kVariants[0])); ++i) {
    const Variant& v = kVariants[i];
    if (v.nseg_h == nseg_h && v.rps_h == rps_h && v.nseg_f == nseg_f && v.rps_f == rps_f && v.head_dim == head_dim &&
        v.bm == bm && v.qkn == qkn && v.dyn == dyn && v.tp == tp)
      return i;
  }
  return -1;
}

const void* decode_kernel_ptr(int variant) { return kFns[variant]; }

size_t decode_smem_bytes(int variant) {
  const bool tc = variant >= 0 && kVariants[variant].bm > kMaxDecodeBatch;
  return ring_bytes(tc) + sizeof(DSmem) + 1024;  // + alignment of the ring to 1024 bytes
}

int launch_decode(int variant, const DecodeParams& p, int grid, cudaStream_t stream, std::string* err) {
  const void* fn = kFns[variant];
  const size_t smem = decode_smem_bytes(variant);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    void* args[] = {const_cast<DecodeParams*>(&p)};
    const bool tc = kVariants[variant].bm > kMaxDecodeBatch;
    e = cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(tc ? kTcBlockThreads : kBlockThreads), args, smem, stream);
  }
  if (e != cudaSuccess) {
    *err = std::string("decode launch: ") + cudaGetErrorString(e);
    return e == cudaErrorCooperativeLaunchTooLarge ? MK_ERR_NOT_RESIDENT : MK_ERR_CUDA;
  }
  return MK_OK;
}

int launch_decode_tp(int variant, const DecodeParams* views, int n_ranks, int sms_per_rank, cudaStream_t stream,
                     std::string* err) {
  if (variant < 0 || !kVariants[variant].tp || n_ranks < 1 || n_ranks > kMaxTpRanks || sms_per_rank < 1) {
    *err = "no tensor-parallel kernel instantiation for this launch";
    return MK_ERR_UNSUPPORTED;
  }
  DecodeParamsTP T;  // copied by the launch
  std::memset(&T, 0, sizeof(T));
  for (int r = 0; r < n_ranks; ++r) T.r[r] = views[r];
  T.sms_per_rank = sms_per_rank;
  const void* fn = kFns[variant];
  const size_t smem = decode_smem_bytes(variant);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    void* args[] = {&T};
    e = cudaLaunchCooperativeKernel(fn, dim3(n_ranks * sms_per_rank), dim3(kBlockThreads), args, smem, stream);
  }
  if (e != cudaSuccess) {
    *err = std::string("tensor-parallel decode launch: ") + cudaGetErrorString(e);
    return e == cudaErrorCooperativeLaunchTooLarge ? MK_ERR_NOT_RESIDENT : MK_ERR_CUDA;
  }
  return MK_OK;
}

}  // namespace mk
