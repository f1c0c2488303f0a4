// mk_attention.cu -- standalone decode attention O = softmax(scale * Q K) V on sm_100a.
//
// The op of the Mirage article's attention example (iaiol.com, "Use Mirage to generate GPU
// kernels for attention": Q [64,1,128], K [64,128,4096] already transposed, V [64,4096,128],
// fp16) with FlashDecoding-style split-KV, which the same article names among the designs
// its search covers.  fp32 accumulation and softmax.
//
// Work split: the keys of all heads form BH * ceil(L/64) units of 64 keys; CTA c of G takes
// units [c*U/G, (c+1)*U/G), so every SM streams the same number of bytes.  A TMA producer
// warp keeps a 6-stage ring of (K^T tile [d][64], V tile [64][d]) fp16 tiles full; eight
// compute warps turn each tile into scores, update a running (max, sum, acc) and, when a
// head's units end inside the CTA, write one partial.  The last CTA to finish a head
// (atomic arrival count) merges that head's partials and resets the count to zero.
//
// L % 8 != 0 cannot be described to TMA (row stride must be a multiple of 16 bytes); those
// shapes take a plain-load kernel (attention_plain) that needs no workspace.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "mk_internal.h"
#include "mk_ptx.cuh"

namespace mk {
namespace attn {

constexpr int kUnit = 64;             // keys per unit
constexpr int kStages = 6;
constexpr int kComputeWarps = 8;
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + producer warp
constexpr int kMaxD = 128;

struct Params {
  const __half_raw* q;  // [BH][d]
  float* o;             // [BH][d]
  float* part;          // [BH][maxc][d + 2]
  uint32_t* cnt;        // [BH] arrival counts, zero between calls
  uint32_t* err;        // error word: 0 = ok, else 1 + stage of the wait that ran out
  int BH, d, L, nu, U, G, maxc;
  float scale;
  uint64_t timeout_ns;
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

struct Smem {
  alignas(128) uint16_t kt[kStages][kMaxD * kUnit];  // [d][64]
  alignas(128) uint16_t v[kStages][kUnit * kMaxD];   // [64][d]
  float red[kComputeWarps][kUnit];                   // partial scores per warp
  float p[kUnit];                                    // probabilities of the current tile
  float acc_red[2048];                               // final per-key-group accumulators [VKG][d]
  float alpha;                                       // rescale factor of the current tile
  float m, l;                                        // running max / sum (warp 0 owns)
  uint32_t last;                                     // this CTA merges head `last` when set
  volatile uint32_t abort;                           // a wait ran out: every role stops waiting
  uint32_t cabort;  // compute-role copy: written only before, and read only after, a compute barrier
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

__device__ __forceinline__ void report_timeout(uint32_t* err, uint32_t code, volatile uint32_t* abort) {
  *abort = 1u;
  atomicCAS(err, 0u, code);
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
      mbar_init(&S.empty[s], kComputeWarps);
    }
    S.abort = 0;
    S.cabort = 0;
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
        mbar_arrive_expect_tx(&S.full[stage], 2u * D * kUnit * 2u);
        tma_load_3d(S.kt[stage], &map_k, j0, 0, h, &S.full[stage], pol);
        tma_load_3d(S.v[stage], &map_v, 0, j0, h, &S.full[stage], pol);
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
  constexpr int DG = D / 32;  // dims per thread in the score phase (4 or 2)
  const int kg = tid & 7;     // score phase: 8-key group
  const int dg = tid >> 3;    // score phase: dim group (0..31)
  const int vdg = tid & (D / 8 - 1);  // PV phase: 8-dim group
  const int vkg = tid / (D / 8);      // PV phase: key group
  constexpr int VKG = 256 / (D / 8);  // key groups in PV phase (16 or 32)
  constexpr int VK = kUnit / VKG;     // keys per thread in PV phase (4 or 2)

  float qreg[DG];
  float acc[8];
  int stage = 0;
  uint32_t phase = 0;
  int cur_h = -1;

  auto begin_head = [&](int h) {
    cur_h = h;
#pragma unroll
    for (int i = 0; i < DG; ++i) qreg[i] = h2f(((const uint16_t*)P.q)[(size_t)h * D + dg * DG + i]) * P.scale;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (tid == 0) {
      S.m = -INFINITY;
      S.l = 0.f;
    }
  };

  auto finish_head = [&]() {
    // reduce acc over key groups, write this CTA's partial for head cur_h, count arrival
#pragma unroll
    for (int i = 0; i < 8; ++i) S.acc_red[vkg * D + vdg * 8 + i] = acc[i];
    named_bar_sync(1, 256);
    const int h = cur_h;
    const int cf = unit_owner(h * P.nu, P.U, P.G);
    const int slot = c - cf;
    float* part = P.part + ((size_t)h * P.maxc + slot) * (D + 2);
    if (tid < D) {
      float s = 0.f;
      for (int g = 0; g < VKG; ++g) s += S.acc_red[g * D + tid];
      part[2 + tid] = s;
    }
    if (tid == 0) {
      part[0] = S.m;
      part[1] = S.l;
    }
    named_bar_sync(1, 256);
    if (tid == 0) {
      __threadfence();
      const int cl = unit_owner((h + 1) * P.nu - 1, P.U, P.G);
      const uint32_t n = (uint32_t)(cl - cf + 1);
      const uint32_t old = atom_acq_rel_gpu_add(&P.cnt[h], 1u);
      S.last = (old + 1 == n) ? n : 0u;
      if (old + 1 == n) P.cnt[h] = 0u;  // self-cleaning for the next call
    }
    named_bar_sync(1, 256);
    if (S.last) {
      __threadfence();
      const int n = (int)S.last;
      const float* base = P.part + (size_t)h * P.maxc * (D + 2);
      if (tid < D) {
        float M = -INFINITY;
        for (int i = 0; i < n; ++i) M = fmaxf(M, __ldcg(base + (size_t)i * (D + 2)));
        float num = 0.f, den = 0.f;
        for (int i = 0; i < n; ++i) {
          const float* pi = base + (size_t)i * (D + 2);
          const float w = expf(__ldcg(pi) - M);
          den += w * __ldcg(pi + 1);
          num += w * __ldcg(pi + 2 + tid);
        }
        P.o[(size_t)h * D + tid] = num / den;
      }
    }
    named_bar_sync(1, 256);
  };

  for (int u = u0; u < u1; ++u) {
    const int h = u / P.nu, j0 = (u % P.nu) * kUnit;
    if (h != cur_h) {
      if (cur_h >= 0) finish_head();
      begin_head(h);
    }
    const int valid = min(kUnit, P.L - j0);
    if (!wait_bar(&S.full[stage], phase, P.timeout_ns, &S.abort)) {
      report_timeout(P.err, 2u, &S.abort);
      S.cabort = 1u;  // every compute thread reaches the barrier below, then all leave together
    }
    // scores: thread (kg, dg) covers keys kg*8..+8 over dims dg*DG..+DG
    const uint16_t* kt = S.kt[stage];
    float sc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sc[j] = 0.f;
#pragma unroll
    for (int i = 0; i < DG; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(kt + (dg * DG + i) * kUnit + kg * 8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2_raw hr;
        hr.x = (unsigned short)(ws[j] & 0xffffu);
        hr.y = (unsigned short)(ws[j] >> 16);
        const float2 f = __half22float2(__half2(hr));
        sc[2 * j] = fmaf(qreg[i], f.x, sc[2 * j]);
        sc[2 * j + 1] = fmaf(qreg[i], f.y, sc[2 * j + 1]);
      }
    }
    // reduce over the 4 dim groups inside the warp (lanes differing in bits 3,4)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sc[j] += __shfl_xor_sync(0xffffffffu, sc[j], 8);
      sc[j] += __shfl_xor_sync(0xffffffffu, sc[j], 16);
    }
    if (lane < 8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) S.red[warp][lane * 8 + j] = sc[j];
    }
    named_bar_sync(1, 256);
    if (S.cabort) return;  // uniform: cabort only changes before this barrier
    if (warp == 0) {
      // lane owns keys lane and lane+32
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        s0 += S.red[w][lane];
        s1 += S.red[w][lane + 32];
      }
      if (lane >= valid) s0 = -INFINITY;
      if (lane + 32 >= valid) s1 = -INFINITY;
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = S.m;
      const float m_new = fmaxf(m_old, mx);
      const float p0 = expf(s0 - m_new), p1 = expf(s1 - m_new);
      float ps = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      S.p[lane] = p0;
      S.p[lane + 32] = p1;
      __syncwarp();
      if (lane == 0) {
        const float a = expf(m_old - m_new);  // 0 on the first tile (m_old = -inf)
        S.alpha = a;
        S.l = S.l * a + ps;
        S.m = m_new;
      }
    }
    named_bar_sync(1, 256);
    // PV: thread (vkg, vdg) covers keys vkg*VK..+VK over dims vdg*8..+8
    const float a = S.alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= a;
    const uint16_t* vt = S.v[stage];
#pragma unroll
    for (int jj = 0; jj < VK; ++jj) {
      const int j = vkg * VK + jj;
      const float p = S.p[j];
      const uint4 w = *reinterpret_cast<const uint4*>(vt + j * D + vdg * 8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2_raw hr;
        hr.x = (unsigned short)(ws[e] & 0xffffu);
        hr.y = (unsigned short)(ws[e] >> 16);
        const float2 f = __half22float2(__half2(hr));
        acc[2 * e] = fmaf(p, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(p, f.y, acc[2 * e + 1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[stage]);
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
  if (cur_h >= 0) finish_head();
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

int attention_decode(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, float* o, int BH, int d, int L,
                     float scale, void* workspace, cudaStream_t stream, int n_sms, uint64_t timeout_ns,
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
  P.q = reinterpret_cast<const __half_raw*>(q);
  P.o = o;
  P.part = reinterpret_cast<float*>(workspace);
  size_t part = (size_t)BH * maxc * (d + 2) * sizeof(float);
  part = (part + 255) & ~(size_t)255;
  P.cnt = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) + part);
  P.err = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) +
                                      attention_error_word_offset(BH, d, L, n_sms));
  P.timeout_ns = timeout_ns;
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
// device.  For them the scratch of the split-KV attention (per-head partials, arrival counts,
// error word) lives in one fixed array in the library's device image instead of a caller
// buffer.  Every GPU that loads the library holds the array until the process exits.
constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB
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
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices ||
      cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    *err = "no usable CUDA device";
    return MK_ERR_CUDA;
  }
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
  if (L % 8 == 0) {
    // the array keeps the previous call's contents: zero the arrival counts and error word
    const size_t counters = attention_counter_offset(BH, d, L, n_sms);
    const cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(scratch) + counters, 0, need - counters, stream);
    if (e != cudaSuccess) {
      *err = std::string("clearing the noalloc counters: ") + cudaGetErrorString(e);
      return MK_ERR_CUDA;
    }
  }
  return attention_decode(q, k_t, v, o, BH, d, L, scale, scratch, stream, n_sms, 2000000000ull, err);
}

}  // namespace mk
