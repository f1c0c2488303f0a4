// mk_attention.cu -- standalone decode attention O = softmax(scale * Q K) V on sm_100a.
//
// The op of the Mirage article's attention example (iaiol.com, "Use Mirage to generate GPU
// kernels for attention": Q [64,1,128], K [64,128,4096] already transposed, V [64,4096,128],
// fp16) with FlashDecoding-style split-KV, which the same article names among the designs
// its search covers.  fp32 accumulation and softmax.
//
// Work split: the keys of all heads form BH * ceil(L/128) units of 128 keys; CTA c of G takes
// units [c*U/G, (c+1)*U/G), so every SM streams the same number of bytes.  A TMA producer
// warp keeps a 3-stage ring of (K^T tile [d][128], V tile [128][d]) fp16 tiles full, in unit
// order (a K^T tile is d rows of 256 contiguous bytes).  The eight compute warps work
// independently and never wait for each other: warp pair p takes units u0 + p, u0 + p + 4, ...,
// warp 2p + h the unit's key half h, each warp with its own running (max, sum, acc) -- lane l
// scores keys 64h + 2l, 64h + 2l + 1 over all d, then owns d/32 output dims in P.V -- and
// both warps of the pair release the stage they read.  At the end of its units of a
// head a warp leaves its partial in a shared-memory slot of the head and goes on (it already
// loaded the next head's q); the last of the head's warps to arrive combines the slot into one
// partial per (CTA, head), written out directly if the head lies inside the CTA, else merged by
// the last CTA to finish the head (atomic arrival count, reset to zero by that CTA).
//
// L % 8 != 0 cannot be described to TMA (row stride must be a multiple of 16 bytes); those
// shapes take a plain-load kernel (attention_plain) that needs no workspace.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <climits>
#include <mutex>

#include "mk_internal.h"
#include "mk_ptx.cuh"

namespace mk {
namespace attn {

constexpr int kUnit = 128;            // keys per unit (one ring stage): 256-byte K^T rows
constexpr int kStages = 3;
constexpr int kComputeWarps = 8;
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + producer warp
constexpr int kMaxD = 128;

struct Params {
  const uint16_t* q;    // [BH][d] fp16
  float* o;             // [BH][d]
  float* part;          // [BH][maxc][d + 2]: per-(head, CTA) partials (m, l, acc[d])
  uint32_t* cnt;        // [BH] arrival counts, zero between calls
  uint32_t* err;        // error word: 0 = ok, else the role of the first wait that ran out
                        // (1 producer slot, 2 tile arrival, 3 combine slot)
  int BH, d, L, nu, U, G, maxc;
  float scale;
  uint64_t timeout_ns;
  int drop_unit;        // test hook: the producer never loads this unit (-1 = none)
};

__host__ __device__ inline int unit_begin(int c, int U, int G) { return (int)(((long long)c * U) / G); }

// CTA that owns unit u (inverse of unit_begin).
__host__ __device__ inline int unit_owner(int u, int U, int G) {
  int c = (int)(((long long)u * G) / U);
  while (c + 1 < G && unit_begin(c + 1, U, G) <= u) ++c;
  while (c > 0 && unit_begin(c, U, G) > u) --c;
  return c;
}

__device__ __forceinline__ float h2f(uint16_t h) {
  __half_raw r;
  r.x = h;
  return __half2float(__half(r));
}

__device__ __forceinline__ float2 h2f2(uint32_t w) {
  __half2_raw r;
  r.x = (unsigned short)(w & 0xffffu);
  r.y = (unsigned short)(w >> 16);
  return __half22float2(__half2(r));
}

struct Smem {
  alignas(128) uint16_t kt[kStages][kMaxD * kUnit];  // [d][128 keys]
  alignas(128) uint16_t v[kStages][kUnit * kMaxD];   // [128 keys][d]
  alignas(16) float qs[kComputeWarps][kMaxD];        // each warp's scaled q of its current head
  alignas(16) float ps[kComputeWarps][kUnit];        // each warp's probabilities of its current unit
  // per-head combine slots (double-buffered by head parity): every warp that took units of the
  // head leaves its (m, l, acc) here; the last one to arrive combines them
  float cm[2][kComputeWarps], cl[2][kComputeWarps];
  alignas(16) float cacc[2][kComputeWarps][kMaxD];
  uint32_t ccount[2];    // warps that left their partial in the slot
  int cowner[2];         // head that owns the slot (-1: free)
  volatile uint32_t abort;  // a wait ran out: every role stops waiting
  // unit whose tiles the producer armed stage s for.  Eight warps take units round-robin over
  // the ring's stages, so a warp can reach a stage's next use before the previous use's tiles
  // have landed; a parity wait cannot tell those phases apart.  A warp first waits until its
  // stage is armed for its unit (the previous use is then complete), then on the stage's phase.
  uint32_t armed[kStages];
  alignas(8) uint64_t full[kStages];
  alignas(8) uint64_t empty[kStages];
};

// Bounded wait on an mbarrier phase: false once `limit_ns` passed or another role aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                         volatile uint32_t* abort) {
  uint64_t t0 = 0;
  for (uint32_t n = 1;; ++n) {
    if (mbar_test(bar, parity)) return true;
    if ((n & 255u) == 0) {
      if (abort && *abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) return false;
    }
  }
}

// Bounded wait until *word == want (acquire): false once `limit_ns` passed or another role
// aborted.
__device__ __forceinline__ bool wait_word(uint32_t* word, uint32_t want, uint64_t limit_ns, volatile uint32_t* abort) {
  uint64_t t0 = 0;
  for (uint32_t n = 1;; ++n) {
    if (ld_acquire_cta_shared(word) == want) return true;
    if ((n & 255u) == 0) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) return false;
    }
  }
}

__device__ __forceinline__ void report_timeout(uint32_t* err, uint32_t code, volatile uint32_t* abort) {
  *abort = 1u;
  atomicCAS(err, 0u, code);
}

// End of a warp's units of head h in this CTA: leave its partial in the head's combine slot.
// The last of the head's contributing warps (nw of them, the first being warp w0) combines the
// slot into one partial per (CTA, head): written out directly if the head lies inside this CTA,
// else stored for the cross-CTA merge, which the last CTA to finish the head performs.  Warp-
// uniform; false if the slot wait ran out.
template <int D>
__device__ __forceinline__ bool flush_head(const Params& P, Smem& S, int h, int c, int w0, int nw, float m, float l,
                                           const float (&acc)[D / 32], int warp, int lane) {
  constexpr int DL = D / 32;
  const int sl = h & 1;
  // claim the slot for head h (free, or already claimed by another warp of this head)
  {
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
      int own = -1;
      if (lane == 0) {
        own = atomicCAS(&S.cowner[sl], -1, h);
      }
      own = __shfl_sync(0xffffffffu, own, 0);
      if (own == -1 || own == h) {
        __threadfence_block();  // the previous owner's reset of the count is seen
        break;
      }
      if ((n & 15u) == 0) {
        if (S.abort) return false;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > P.timeout_ns) return false;
      }
    }
  }
  if (lane == 0) {
    S.cm[sl][warp] = m;
    S.cl[sl][warp] = l;
  }
#pragma unroll
  for (int i = 0; i < DL; ++i) S.cacc[sl][warp][lane * DL + i] = acc[i];
  __syncwarp();
  uint32_t arrived = 0;
  if (lane == 0) {
    __threadfence_block();
    arrived = atomicAdd(&S.ccount[sl], 1u) + 1u;
  }
  arrived = __shfl_sync(0xffffffffu, arrived, 0);
  if (arrived != (uint32_t)nw) return true;
  // this warp combines: every contributing warp's writes are visible (fence + atomic)
  __threadfence_block();
  float M = -INFINITY;
  for (int k = 0; k < nw; ++k) M = fmaxf(M, S.cm[sl][(w0 + k) & (kComputeWarps - 1)]);
  float ls = 0.f, as[DL];
#pragma unroll
  for (int i = 0; i < DL; ++i) as[i] = 0.f;
  for (int k = 0; k < nw; ++k) {
    const int w = (w0 + k) & (kComputeWarps - 1);
    const float f = __expf(S.cm[sl][w] - M);
    ls = fmaf(f, S.cl[sl][w], ls);
#pragma unroll
    for (int i = 0; i < DL; ++i) as[i] = fmaf(f, S.cacc[sl][w][lane * DL + i], as[i]);
  }
  // the slot is read: free it for head h + 2
  __syncwarp();
  if (lane == 0) {
    S.ccount[sl] = 0u;
    __threadfence_block();
    atomicExch(&S.cowner[sl], -1);
  }
  const int cf = unit_owner(h * P.nu, P.U, P.G), cl = unit_owner((h + 1) * P.nu - 1, P.U, P.G);
  if (cf == cl) {  // the head lies inside this CTA
#pragma unroll
    for (int i = 0; i < DL; ++i) P.o[(size_t)h * D + lane * DL + i] = as[i] / ls;
    return true;
  }
  float* part = P.part + ((size_t)h * P.maxc + (c - cf)) * (D + 2);
#pragma unroll
  for (int i = 0; i < DL; ++i) part[2 + lane * DL + i] = as[i];
  if (lane == 0) {
    part[0] = M;
    part[1] = ls;
  }
  __syncwarp();
  uint32_t last = 0;
  const uint32_t n = (uint32_t)(cl - cf + 1);
  if (lane == 0) {
    __threadfence();
    const uint32_t old = atom_acq_rel_gpu_add(&P.cnt[h], 1u);
    last = (old + 1 == n) ? 1u : 0u;
    if (last) P.cnt[h] = 0u;  // self-cleaning for the next call
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return true;
  // the last CTA of the head merges every CTA's partial, eight per L2 round trip
  __threadfence();
  const float* base = P.part + (size_t)h * P.maxc * (D + 2);
  float M2 = -INFINITY;
  for (int i = 0; i < (int)n; ++i) M2 = fmaxf(M2, ldcg_f32(base + (size_t)i * (D + 2)));
  float num[DL], den = 0.f;
#pragma unroll
  for (int i = 0; i < DL; ++i) num[i] = 0.f;
  for (int i0 = 0; i0 < (int)n; i0 += 8) {
    float mv[8], lv[8], av[8][DL];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool in = i0 + k < (int)n;
      const float* pi = base + (size_t)(in ? i0 + k : 0) * (D + 2);
      mv[k] = in ? ldcg_f32(pi) : -INFINITY;
      lv[k] = in ? ldcg_f32(pi + 1) : 0.f;
#pragma unroll
      for (int i = 0; i < DL; ++i) av[k][i] = in ? ldcg_f32(pi + 2 + lane * DL + i) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float f = (mv[k] == -INFINITY) ? 0.f : __expf(mv[k] - M2);
      den = fmaf(f, lv[k], den);
#pragma unroll
      for (int i = 0; i < DL; ++i) num[i] = fmaf(f, av[k][i], num[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < DL; ++i) P.o[(size_t)h * D + lane * DL + i] = num[i] / den;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attention_split_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                           Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int u0 = unit_begin(c, P.U, P.G), u1 = unit_begin(c + 1, P.U, P.G);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 2);  // the warp pair that read the stage releases it
      S.armed[s] = 0xffffffffu;
    }
    for (int s = 0; s < 2; ++s) {
      S.ccount[s] = 0u;
      S.cowner[s] = -1;
    }
    S.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      const uint64_t pol = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int u = u0; u < u1; ++u) {
        const int h = u / P.nu, j0 = (u % P.nu) * kUnit;
        if (!wait_bar(&S.empty[stage], phase ^ 1, P.timeout_ns, &S.abort)) {
          report_timeout(P.err, 1u, &S.abort);
          break;
        }
        if (u != P.drop_unit) {
          mbar_arrive_expect_tx(&S.full[stage], 2u * D * kUnit * 2u);
          tma_load_3d(S.kt[stage], &map_k, j0, 0, h, &S.full[stage], pol);
          tma_load_3d(S.v[stage], &map_v, 0, j0, h, &S.full[stage], pol);
          st_release_cta_shared(&S.armed[stage], (uint32_t)u);  // the stage's previous use is released
        }
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last issued stages to land.
      for (int i = 1; i <= (issued < kStages ? issued : kStages); ++i) {
        int s = stage - i, ph = (int)phase;
        if (s < 0) {
          s += kStages;
          ph ^= 1;
        }
        wait_bar(&S.full[s], (uint32_t)ph, P.timeout_ns, nullptr);
      }
    }
    return;
  }

  // ---------------- compute warps ----------------
  // Warp pair p (warps 2p, 2p + 1) takes units u0 + p, u0 + p + 4, ... (heads in order); warp
  // 2p + h takes key half h of each, with its own running (max, sum, acc), so a stage is held
  // for half the time one warp would need.  At the end of its units of a head a warp leaves
  // its partial in the head's combine slot (flush_head) and goes on.  No compute-warp barrier:
  // a wait that runs out makes the warp skip its remaining work.
  constexpr int DL = D / 32;  // output dims per lane in P.V
  constexpr int KPW = kUnit / 2;  // keys per warp (half a unit)
  constexpr int KPL = KPW / 32;   // keys per lane in the scores (2)
  constexpr int kPairs = kComputeWarps / 2;
  const int kb = (warp & 1) * KPW;  // this warp's first key of a unit
  float* qs = S.qs[warp];
  float* ps = S.ps[warp];
  bool alive = true;
  int cur_h = -1;
  float m = -INFINITY, l = 0.f, acc[DL];
  float qn[DL];  // the next head's q (prefetched)
  auto flush = [&](int h) {
    const int a = max(u0, h * P.nu), b = min(u1, (h + 1) * P.nu);  // the head's units in this CTA
    // the head's warps: both warps of every pair that took one of its units
    const int nw = 2 * min(kPairs, b - a), w0 = 2 * ((a - u0) & (kPairs - 1));
    if (alive && !flush_head<D>(P, S, h, c, w0, nw, m, l, acc, warp, lane)) {
      if (lane == 0) report_timeout(P.err, 3u, &S.abort);
      alive = false;
    }
  };
  for (int u = u0 + (warp >> 1); u < u1 && alive; u += kPairs) {
    const int h = u / P.nu;
    if (h != cur_h) {
      if (cur_h >= 0) flush(cur_h);
      if (cur_h < 0) {  // the first head's q (later heads were prefetched)
        const uint16_t* qh = P.q + (size_t)h * D + lane * DL;
#pragma unroll
        for (int i = 0; i < DL; ++i) qn[i] = h2f(__ldg(qh + i)) * P.scale;
      }
#pragma unroll
      for (int i = 0; i < DL; ++i) qs[lane * DL + i] = qn[i];
      __syncwarp();
      // the q of the head after this one, loaded while this one runs
      {
        const int hn = min(h + 1, P.BH - 1);
        const uint16_t* qh = P.q + (size_t)hn * D + lane * DL;
#pragma unroll
        for (int i = 0; i < DL; ++i) qn[i] = h2f(__ldg(qh + i)) * P.scale;
      }
      cur_h = h;
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int i = 0; i < DL; ++i) acc[i] = 0.f;
    }
    const int idx = u - u0, stage = idx % kStages;
    const uint32_t parity = (uint32_t)(idx / kStages) & 1u;
    bool ok = wait_word(&S.armed[stage], (uint32_t)u, P.timeout_ns, &S.abort) &&
              wait_bar(&S.full[stage], parity, P.timeout_ns, &S.abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) report_timeout(P.err, 2u, &S.abort);
      alive = false;
      break;
    }
    const int valid = min(KPW, min(kUnit, P.L - (u % P.nu) * kUnit) - kb);  // this warp's keys
    if (valid <= 0) {  // warp-uniform: the unit's second half lies past L
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[stage]);
      continue;
    }
    // scores: lane owns keys kb + KPL*lane .. + KPL-1; row dd of the K^T tile holds 128 keys
    const uint16_t* kt = S.kt[stage] + kb + lane * KPL;
    float sa[KPL], sb[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) sa[k] = sb[k] = 0.f;
#pragma unroll 4
    for (int dd = 0; dd < D; dd += 4) {
      const float4 q4 = *reinterpret_cast<const float4*>(qs + dd);
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 k01 = h2f2(*reinterpret_cast<const uint32_t*>(kt + (dd + e) * kUnit));
        float* s = (e & 1) ? sb : sa;
        s[0] = fmaf(qv[e], k01.x, s[0]);
        s[1] = fmaf(qv[e], k01.y, s[1]);
      }
    }
    float sc[KPL], bm = -INFINITY;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      sc[k] = (lane * KPL + k < valid) ? sa[k] + sb[k] : -INFINITY;
      bm = fmaxf(bm, sc[k]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    const float m_new = fmaxf(m, bm);  // finite: the warp's half holds at least one key
    const float alpha = __expf(m - m_new);  // 0 on the head's first unit (m = -inf)
    float p[KPL], psum = 0.f;
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
      p[k] = __expf(sc[k] - m_new);
      psum += p[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = fmaf(l, alpha, psum);
    m = m_new;
#pragma unroll
    for (int i = 0; i < DL; ++i) acc[i] *= alpha;
    *reinterpret_cast<float2*>(ps + KPL * lane) = make_float2(p[0], p[1]);
    __syncwarp();
    // P.V: lane owns dims lane*DL .. lane*DL + DL - 1 (keys past L have p = 0 and zero rows)
    const uint16_t* vt = S.v[stage] + (size_t)kb * D + lane * DL;
#pragma unroll 4
    for (int k = 0; k < KPW; k += 4) {
      const float4 p4 = *reinterpret_cast<const float4*>(ps + k);
      const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (DL == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(vt + (k + e) * D);
          const float2 a = h2f2(w.x), b = h2f2(w.y);
          acc[0] = fmaf(pv[e], a.x, acc[0]);
          acc[1] = fmaf(pv[e], a.y, acc[1]);
          acc[2] = fmaf(pv[e], b.x, acc[2]);
          acc[3] = fmaf(pv[e], b.y, acc[3]);
        } else {
          const float2 a = h2f2(*reinterpret_cast<const uint32_t*>(vt + (k + e) * D));
          acc[0] = fmaf(pv[e], a.x, acc[0]);
          acc[1] = fmaf(pv[e], a.y, acc[1]);
        }
      }
    }
    __syncwarp();  // every lane's reads of the stage and of ps are done
    if (lane == 0) mbar_arrive(&S.empty[stage]);
  }
  if (alive && cur_h >= 0) flush(cur_h);
}

// Plain-load path for any L: one CTA per head, scores staged in shared memory in chunks.
__global__ void __launch_bounds__(256) attention_plain(const uint16_t* q, const uint16_t* kt, const uint16_t* v,
                                                       float* o, int d, int L, float scale) {
  __shared__ float qs[kMaxD];
  __shared__ float sc[1024];
  __shared__ float red[8];
  __shared__ float accs[2][kMaxD];
  const int h = blockIdx.x, tid = threadIdx.x;
  if (tid < d) qs[tid] = h2f(q[(size_t)h * d + tid]) * scale;
  float m = -INFINITY, l = 0.f, acc = 0.f;  // thread tid < d owns acc for dim tid; others idle in PV
  const int half = tid >> 7, dd = tid & 127;
  __syncthreads();
  for (int j0 = 0; j0 < L; j0 += 1024) {
    const int n = min(1024, L - j0);
    float lmax = -INFINITY;
    for (int j = tid; j < n; j += 256) {
      float s = 0.f;
      for (int t = 0; t < d; ++t) s = fmaf(qs[t], h2f(kt[((size_t)h * d + t) * L + j0 + j]), s);
      sc[j] = s;
      lmax = fmaxf(lmax, s);
    }
    for (int off = 16; off > 0; off >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, off));
    if ((tid & 31) == 0) red[tid >> 5] = lmax;
    __syncthreads();
    float cmax = red[0];
    for (int w = 1; w < 8; ++w) cmax = fmaxf(cmax, red[w]);
    const float m_new = fmaxf(m, cmax);
    const float a = expf(m - m_new);
    __syncthreads();
    float ls = 0.f;
    for (int j = tid; j < n; j += 256) {
      const float p = expf(sc[j] - m_new);
      sc[j] = p;
      ls += p;
    }
    for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
    if ((tid & 31) == 0) red[tid >> 5] = ls;
    __syncthreads();
    float csum = 0.f;
    for (int w = 0; w < 8; ++w) csum += red[w];
    l = l * a + csum;
    m = m_new;
    acc *= a;
    if (dd < d) {
      // the two halves of the block split the keys of this chunk
      for (int j = half; j < n; j += 2) acc = fmaf(sc[j], h2f(v[((size_t)h * L + j0 + j) * d + dd]), acc);
    }
    __syncthreads();
  }
  if (dd < d) accs[half][dd] = acc;
  __syncthreads();
  if (tid < d) o[(size_t)h * d + tid] = (accs[0][tid] + accs[1][tid]) / l;
}

}  // namespace attn

static int attn_geometry(int BH, int d, int L, int n_sms, int* nu, int* U, int* G, int* maxc) {
  *nu = (L + attn::kUnit - 1) / attn::kUnit;
  *U = BH * (*nu);
  *G = n_sms < *U ? n_sms : *U;
  // contributors per head: CTAs whose unit range meets the head's units
  int m = 1;
  for (int h = 0; h < BH; ++h) {
    int cf = attn::unit_owner(h * (*nu), *U, *G), cl = attn::unit_owner((h + 1) * (*nu) - 1, *U, *G);
    if (cl - cf + 1 > m) m = cl - cf + 1;
  }
  *maxc = m;
  (void)d;
  return 0;
}

size_t attention_workspace_bytes(int BH, int d, int L, int n_sms) {
  if (BH < 1 || L < 1 || (d != 64 && d != 128)) return 0;
  int nu, U, G, maxc;
  attn_geometry(BH, d, L, n_sms, &nu, &U, &G, &maxc);
  size_t part = (size_t)BH * maxc * (d + 2) * sizeof(float);
  part = (part + 255) & ~(size_t)255;
  return part + (((size_t)BH * sizeof(uint32_t) + 255) & ~(size_t)255) + 256;
}

size_t attention_counter_offset(int BH, int d, int L, int n_sms) {
  int nu, U, G, maxc;
  attn_geometry(BH, d, L, n_sms, &nu, &U, &G, &maxc);
  return ((size_t)BH * maxc * (d + 2) * sizeof(float) + 255) & ~(size_t)255;
}

size_t attention_error_word_offset(int BH, int d, int L, int n_sms) {
  return attention_workspace_bytes(BH, d, L, n_sms) - 256;
}

static bool encode_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                       uint32_t b1) {
  auto fn = get_tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
std::atomic<uint64_t> g_attn_timeout_ns{2000000000ull};  // limit of every device wait
std::atomic<int> g_attn_drop_unit{-1};                   // test hook (see mk_attention_debug_drop_unit)
}  // namespace

void attention_set_wait_timeout_ns(uint64_t ns) { g_attn_timeout_ns.store(ns); }
void attention_debug_drop_unit(int unit) { g_attn_drop_unit.store(unit); }

int attention_decode(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d, int L,
                     float scale, void* workspace, cudaStream_t stream, int n_sms, uint32_t* err_word,
                     std::string* err) {
  if (L % 8 != 0) {
    attn::attention_plain<<<BH, 256, 0, stream>>>(q, k_t, v, o, d, L, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *err = std::string("attention_plain launch: ") + cudaGetErrorString(e);
      return MK_ERR_CUDA;
    }
    return MK_OK;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) {
    *err = "workspace must be a 256-byte aligned device pointer";
    return MK_ERR_INVALID_ARG;
  }
  int nu, U, G, maxc;
  attn_geometry(BH, d, L, n_sms, &nu, &U, &G, &maxc);
  attn::Params P;
  P.q = q;
  P.o = o;
  P.part = reinterpret_cast<float*>(workspace);
  P.cnt = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) +
                                      attention_counter_offset(BH, d, L, n_sms));
  P.err = err_word ? err_word
                   : reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) +
                                                 attention_error_word_offset(BH, d, L, n_sms));
  P.timeout_ns = g_attn_timeout_ns.load();
  P.drop_unit = g_attn_drop_unit.load();
  P.BH = BH;
  P.d = d;
  P.L = L;
  P.nu = nu;
  P.U = U;
  P.G = G;
  P.maxc = maxc;
  P.scale = scale;
  CUtensorMap mk_, mv_;
  // K^T: [BH][d][L] -> dims {L, d, BH}, box {64 keys, d dims}
  // V:   [BH][L][d] -> dims {d, L, BH}, box {d dims, 64 keys}
  if (!encode_map(&mk_, k_t, (uint64_t)L, (uint64_t)d, (uint64_t)BH, attn::kUnit, (uint32_t)d) ||
      !encode_map(&mv_, v, (uint64_t)d, (uint64_t)L, (uint64_t)BH, (uint32_t)d, attn::kUnit)) {
    *err = "cuTensorMapEncodeTiled failed for the attention operands (pointer alignment?)";
    return MK_ERR_INVALID_ARG;
  }
  const size_t smem = sizeof(attn::Smem) + 1024;
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(attn::attention_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e == cudaSuccess) attn::attention_split_kernel<128><<<G, attn::kThreads, smem, stream>>>(mk_, mv_, P);
  } else {
    e = cudaFuncSetAttribute(attn::attention_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e == cudaSuccess) attn::attention_split_kernel<64><<<G, attn::kThreads, smem, stream>>>(mk_, mv_, P);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *err = std::string("attention_split launch: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  return MK_OK;
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant.  Some callers may not call cudaMalloc: a serving process whose own
// allocator reserved the device memory up front (a library allocation would fail or fragment
// it), or a latency-critical loop where cudaMalloc/cudaFree would block and synchronise the
// device.  For them the scratch of the split-KV attention (per-head partials, arrival counts)
// lives in one fixed array in the library's device image instead of a caller buffer, and the
// error word in the array's last 256 bytes.  Every GPU that loads the library holds the array
// until the process exits.
constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB
constexpr size_t kNoAllocErrOffset = kNoAllocScratchBytes - 256;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
}  // namespace

size_t attention_noalloc_capacity() { return kNoAllocScratchBytes; }

int attention_decode_noalloc(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d,
                             int L, float scale, cudaStream_t stream, std::string* err) {
  int dev = 0, n_sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    *err = "no usable CUDA device";
    return MK_ERR_CUDA;
  }
  if (dev < 0 || dev >= kNoAllocMaxDevices) {
    *err = "mk_attention_decode_noalloc: device index " + std::to_string(dev) +
           " exceeds the per-device address table (" + std::to_string(kNoAllocMaxDevices) + " devices)";
    return MK_ERR_UNSUPPORTED;
  }
  // the per-call scratch ends with its own 256-byte error slot, which this variant does not
  // use (its error word sits at a fixed place): it fits iff need <= the array's size
  const size_t need = attention_workspace_bytes(BH, d, L, n_sms);
  if (need > kNoAllocScratchBytes) {
    *err = "mk_attention_decode_noalloc: these sizes need " + std::to_string(need) +
           " bytes of scratch; the fixed array holds " + std::to_string(kNoAllocScratchBytes) +
           " (use mk_attention_decode with a caller workspace)";
    return MK_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  {
    // once per device, with that device current: the array's device address (the symbol
    // itself is only a host-side stand-in)
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        *err = std::string("cudaGetSymbolAddress(noalloc scratch): ") + cudaGetErrorString(e);
        return MK_ERR_CUDA;
      }
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  uint8_t* base = static_cast<uint8_t*>(scratch);
  if (L % 8 == 0) {
    // the array keeps the previous call's contents: zero the arrival counts (the error word
    // keeps the first timeout until attention_noalloc_status reads it)
    const size_t counters = attention_counter_offset(BH, d, L, n_sms);
    const cudaError_t e = cudaMemsetAsync(base + counters, 0, need - 256 - counters, stream);
    if (e != cudaSuccess) {
      *err = std::string("clearing the noalloc counters: ") + cudaGetErrorString(e);
      return MK_ERR_CUDA;
    }
  }
  return attention_decode(q, k_t, v, o, BH, d, L, scale, scratch, stream, n_sms,
                          reinterpret_cast<uint32_t*>(base + kNoAllocErrOffset), err);
}

int attention_noalloc_status(cudaStream_t stream, std::string* err) {
  cudaError_t e = cudaStreamSynchronize(stream);
  uint32_t word = 0;
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&word, g_noalloc_scratch, 4, kNoAllocErrOffset, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && word != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_noalloc_scratch, &zero, 4, kNoAllocErrOffset, cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    *err = std::string("reading the noalloc error word: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  if (word != 0) {
    *err = "mk_attention_decode_noalloc: a device wait timed out (its output is undefined)";
    return MK_ERR_DEVICE_TIMEOUT;
  }
  return MK_OK;
}

}  // namespace mk
