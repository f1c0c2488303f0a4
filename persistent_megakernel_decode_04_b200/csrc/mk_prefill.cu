// mk_prefill.cu -- prompt processing on ordinary (non-persistent) kernels.
//
// The hybrid arrangement of "Ada-MK: Adaptive MegaKernel Optimization via Automated
// DAG-based Search for LLM Inference" (section 3, the heterogeneous engine): the prompt runs
// on standard kernels and only decode runs on the megakernel.  Prefill is not the timed
// path; it fills the KV cache and gives the last prompt token's logits.  Tokens are taken
// in chunks of at most rows_cap (sequence, position) rows; each chunk runs every layer.
// Weights are read from the same packed arena the megakernel streams (QKV rows grouped per
// KV head with RoPE pairs adjacent, gate/up rows interleaved).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <string>

#include "mk_internal.h"

namespace mk {
namespace pf {

__device__ __forceinline__ float bf(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// X[row] = E[token] for rows (b, tt) of the chunk, row = b * ct + tt.
__global__ void embed(const int32_t* tokens, int T, int t0, int ct, const uint16_t* E, float* X, int H, int V) {
  const int row = blockIdx.x, b = row / ct, tt = row % ct;
  int tok = tokens[(size_t)b * T + t0 + tt];
  if (tok < 0 || tok >= V) tok = 0;  // out-of-range ids read row 0 instead of outside the table
  for (int i = threadIdx.x; i < H; i += blockDim.x) X[(size_t)row * H + i] = bf(E[(size_t)tok * H + i]);
}

// Y[row] = X[src_row(row)] * rsqrt(mean(x^2) + eps) * g
__global__ void rmsnorm(const float* X, const uint16_t* g, float* Y, int H, float eps, int src_stride_rows,
                        int src_offset_rows) {
  const int row = blockIdx.x;
  const float* x = X + ((size_t)row * src_stride_rows + src_offset_rows) * H;
  __shared__ float red[32];
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(x[i], x[i], ss);
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float r = 1.0f / sqrtf(red[0] / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x) Y[(size_t)row * H + i] = x[i] * r * bf(g[i]);
}

// Element (r, k) of a [N][K] bf16 weight matrix: row-major, or (blocked) in the tensor-core
// layout of kTcRows x kTcUnitK blocks of 8-row x 8-element core matrices.
__device__ __forceinline__ size_t w_index(int r, int k, int K, int blocked) {
  if (!blocked) return (size_t)r * K + k;
  const int nk = (K + kTcUnitK - 1) / kTcUnitK;
  const size_t blk = (size_t)(r / kTcRows) * nk + k / kTcUnitK;
  return blk * (kTcRows * kTcUnitK) + (size_t)(((r % kTcRows) / 8) * (kTcUnitK / 8) + (k % kTcUnitK) / 8) * 64 +
         (r % 8) * 8 + (k % 8);
}

// Y[n][N] (row stride ldy) (+)= A[n][K] (fp32, row stride lda) . W[N][K]^T (bf16), fp32
// accumulation.  64 x 64 output tile per block, 256 threads x (4 x 4) outputs, K tile 32.
constexpr int BM = 64, BN = 64, BK = 32;
__global__ void __launch_bounds__(256) gemm(const float* __restrict__ A, const uint16_t* __restrict__ W,
                                            float* __restrict__ Y, int n, int N, int K, int lda, int ldy,
                                            int accumulate, int blocked) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tx = tid % 16, ty = tid / 16;  // outputs rows ty*4.., cols tx*4..
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    // A tile: 64 rows x 32 k = 2048 floats, 8 per thread
    for (int e = tid; e < BM * BK; e += 256) {
      const int r = e / BK, k = e % BK;
      const int gr = m0 + r, gk = k0 + k;
      As[k][r] = (gr < n && gk < K) ? A[(size_t)gr * lda + gk] : 0.f;
    }
    for (int e = tid; e < BN * BK; e += 256) {
      const int r = e / BK, k = e % BK;
      const int gr = n0 + r, gk = k0 + k;
      Ws[k][r] = (gr < N && gk < K) ? bf(W[w_index(gr, gk, K, blocked)]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < BK; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[k][ty * 4 + i];
        w[i] = Ws[k][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gr = m0 + ty * 4 + i;
    if (gr >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gc = n0 + tx * 4 + j;
      if (gc < N) Y[(size_t)gr * ldy + gc] = accumulate ? Y[(size_t)gr * ldy + gc] + acc[i][j] : acc[i][j];
    }
  }
}

// QK-norm (Mirage article, "Case 4.1: Attention with Query-Key Normalization"): LayerNorm of
// every q and k head of a packed QKV output row, in place, before RoPE.  One block per row, one
// warp per head; a head's D values sit at packed positions 2i (dim i) and 2i + 1 (dim i + D/2).
// Gains and biases: q gain [nq*D], q bias [nq*D], k gain [nkv*D], k bias [nkv*D].
__global__ void qk_norm(float* Yq, const uint16_t* nb, int nq, int nkv, int D, float eps) {
  const int G = nq / nkv, rpg = (G + 2) * D, NQKV = (nq + 2 * nkv) * D, half = D / 2;
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float* y = Yq + (size_t)blockIdx.x * NQKV;
  for (int h = threadIdx.x >> 5; h < nq + nkv; h += nw) {  // heads 0..nq-1: q; then k
    const int grp = h < nq ? h / G : h - nq;
    float* v = y + (size_t)grp * rpg + (h < nq ? (h % G) * D : G * D);
    const uint16_t* g = nb + (h < nq ? (size_t)h * D : (size_t)2 * nq * D + (size_t)(h - nq) * D);
    const uint16_t* b = g + (h < nq ? (size_t)nq * D : (size_t)nkv * D);
    float sum = 0.f;
    for (int e = lane; e < D; e += 32) sum += v[e];
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float mean = sum / D;
    float sq = 0.f;
    for (int e = lane; e < D; e += 32) sq += (v[e] - mean) * (v[e] - mean);
    for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    const float r = 1.0f / sqrtf(sq / D + eps);
    for (int e = lane; e < D; e += 32) {
      const int dim = (e & 1) ? (e >> 1) + half : (e >> 1);
      v[e] = (v[e] - mean) * r * bf(g[dim]) + bf(b[dim]);
    }
  }
}

// Packed QKV output row -> RoPE'd q (natural head/dim order) and bf16 K/V cache entries.
__global__ void qkv_post(const float* Yq, int n, int ct, int t0, const float2* rope, float* Q, uint16_t* kv,
                         int layer, int nq, int nkv, int D, int max_seq, int max_batch) {
  const int row = blockIdx.x, b = row / ct, pos = t0 + row % ct;
  const int G = nq / nkv, half = D / 2, rpg = (G + 2) * D, NQKV = (nq + 2 * nkv) * D;
  const size_t head_stride = (size_t)max_seq * D;
  const size_t kv_layer = (size_t)max_batch * nkv * head_stride;
  const float* y = Yq + (size_t)row * NQKV;
  for (int R = threadIdx.x; R < NQKV; R += blockDim.x) {
    const int grp = R / rpg, rr = R % rpg;
    const float v = y[R];
    if (rr < (G + 1) * D) {
      const int pd = (rr < G * D) ? (rr % D) : (rr - G * D);
      const int i = pd >> 1, hi = pd & 1;
      const float other = y[R ^ 1];
      const float2 cs = rope[(size_t)pos * half + i];
      const float outv = hi ? (v * cs.x + other * cs.y) : (v * cs.x - other * cs.y);
      const int dim = hi ? i + half : i;
      if (rr < G * D) {
        Q[(size_t)row * nq * D + (size_t)(grp * G + rr / D) * D + dim] = outv;
      } else {
        kv[((size_t)layer * 2 + 0) * kv_layer + ((size_t)b * nkv + grp) * head_stride + (size_t)pos * D + dim] =
            f2bf(outv);
      }
    } else {
      const int dim = rr - (G + 1) * D;
      kv[((size_t)layer * 2 + 1) * kv_layer + ((size_t)b * nkv + grp) * head_stride + (size_t)pos * D + dim] =
          f2bf(v);
    }
  }
}

// Causal attention of chunk row (b, pos) and query head h over cache positions 0..pos.
// One block per (row, head); scores staged in dynamic shared memory (pos + 1 floats).
__global__ void __launch_bounds__(128) attention(const float* Q, const uint16_t* kv, float* O, int ct, int t0,
                                                 int layer, int nq, int nkv, int D, int max_seq, int max_batch,
                                                 float scale) {
  extern __shared__ float sc[];
  __shared__ float qs[128];
  __shared__ float red[4];
  const int row = blockIdx.x / nq, h = blockIdx.x % nq;
  const int b = row / ct, pos = t0 + row % ct, L = pos + 1;
  const int kvh = (int)((long long)h * nkv / nq);
  const size_t head_stride = (size_t)max_seq * D;
  const size_t kv_layer = (size_t)max_batch * nkv * head_stride;
  const uint16_t* kc = kv + ((size_t)layer * 2 + 0) * kv_layer + ((size_t)b * nkv + kvh) * head_stride;
  const uint16_t* vc = kv + ((size_t)layer * 2 + 1) * kv_layer + ((size_t)b * nkv + kvh) * head_stride;
  const int tid = threadIdx.x;
  if (tid < D) qs[tid] = Q[(size_t)row * nq * D + (size_t)h * D + tid] * scale;
  __syncthreads();
  float mx = -INFINITY;
  for (int j = tid; j < L; j += 128) {
    const uint4* kr = reinterpret_cast<const uint4*>(kc + (size_t)j * D);
    float s = 0.f;
    for (int v8 = 0; v8 < D / 8; ++v8) {
      const uint4 w = kr[v8];
      const float* q = qs + v8 * 8;
      s = fmaf(q[0], __uint_as_float(w.x << 16), s);
      s = fmaf(q[1], __uint_as_float(w.x & 0xffff0000u), s);
      s = fmaf(q[2], __uint_as_float(w.y << 16), s);
      s = fmaf(q[3], __uint_as_float(w.y & 0xffff0000u), s);
      s = fmaf(q[4], __uint_as_float(w.z << 16), s);
      s = fmaf(q[5], __uint_as_float(w.z & 0xffff0000u), s);
      s = fmaf(q[6], __uint_as_float(w.w << 16), s);
      s = fmaf(q[7], __uint_as_float(w.w & 0xffff0000u), s);
    }
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float ls = 0.f;
  for (int j = tid; j < L; j += 128) {
    const float p = expf(sc[j] - mx);
    sc[j] = p;
    ls += p;
  }
  for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  if ((tid & 31) == 0) red[tid >> 5] = ls;
  __syncthreads();
  const float l = red[0] + red[1] + red[2] + red[3];
  if (tid < D) {
    float a = 0.f;
    for (int j = 0; j < L; ++j) a = fmaf(sc[j], bf(vc[(size_t)j * D + tid]), a);
    O[(size_t)row * nq * D + (size_t)h * D + tid] = a / l;
  }
}

__global__ void residual_add(float* X, const float* Y, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    X[i] += Y[i];
}

// Y rows are interleaved (g_i, u_i); HH[row][i] = silu(g_i) * u_i
__global__ void swiglu(const float* Y, float* HH, int F) {
  const int row = blockIdx.x;
  for (int i = threadIdx.x; i < F; i += blockDim.x) {
    const float g = Y[(size_t)row * 2 * F + 2 * i], u = Y[(size_t)row * 2 * F + 2 * i + 1];
    HH[(size_t)row * F + i] = g / (1.f + expf(-g)) * u;
  }
}

}  // namespace pf

static bool ck(cudaError_t e, const char* what, std::string* err) {
  if (e == cudaSuccess) return true;
  *err = std::string(what) + ": " + cudaGetErrorString(e);
  return false;
}

static void gemm(const float* A, const uint16_t* W, float* Y, int n, int N, int K, int ldy, cudaStream_t s,
                 int blocked, int lda = -1, int accumulate = 0) {
  dim3 grid((N + pf::BN - 1) / pf::BN, (n + pf::BM - 1) / pf::BM);
  pf::gemm<<<grid, 256, 0, s>>>(A, W, Y, n, N, K, lda < 0 ? K : lda, ldy, accumulate, blocked);
}

int run_prefill(const PrefillParams& p, const int32_t* tokens, int B, int T, float* last_logits, cudaStream_t s,
                std::string* err) {
  const int H = p.H, D = p.D, F = p.F, nq = p.nq, nkv = p.nkv;
  const int NQKV = (nq + 2 * nkv) * D;
  const int ct_max = p.rows_cap / B;
  if (ct_max < 1) {
    *err = "prefill scratch too small for this batch";
    return MK_ERR_INVALID_ARG;
  }
  const uint16_t* E = reinterpret_cast<const uint16_t*>(p.arena + p.off_embed);
  int last_t0 = 0, last_ct = 1;
  for (int t0 = 0; t0 < T; t0 += ct_max) {
    const int ct = (T - t0) < ct_max ? (T - t0) : ct_max;
    const int n = B * ct;
    last_t0 = t0;
    last_ct = ct;
    pf::embed<<<n, 256, 0, s>>>(tokens, T, t0, ct, E, p.X, H, p.V);
    for (int l = 0; l < p.L; ++l) {
      const LayerOff& lo = p.loff_host[l];
      const uint16_t* an = reinterpret_cast<const uint16_t*>(p.arena + lo.attn_norm);
      const uint16_t* mn = reinterpret_cast<const uint16_t*>(p.arena + lo.mlp_norm);
      pf::rmsnorm<<<n, 256, 0, s>>>(p.X, an, p.XN, H, p.eps, 1, 0);
      gemm(p.XN, reinterpret_cast<const uint16_t*>(p.arena + lo.qkv), p.Y, n, NQKV, H, NQKV, s, p.blocked);
      if (p.qk_norm)
        pf::qk_norm<<<n, 256, 0, s>>>(p.Y, reinterpret_cast<const uint16_t*>(p.arena + lo.qkn), nq, nkv, D, p.eps);
      pf::qkv_post<<<n, 256, 0, s>>>(p.Y, n, ct, t0, p.rope, p.Q, p.kv, l, nq, nkv, D, p.max_seq, p.max_batch);
      const size_t smem = (size_t)(t0 + ct) * sizeof(float);
      if (smem > 48 * 1024) cudaFuncSetAttribute(pf::attention, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      pf::attention<<<n * nq, 128, smem, s>>>(p.Q, p.kv, p.O, ct, t0, l, nq, nkv, D, p.max_seq, p.max_batch,
                                              p.attn_scale);
      gemm(p.O, reinterpret_cast<const uint16_t*>(p.arena + lo.o), p.Y, n, H, nq * D, H, s, p.blocked);
      pf::residual_add<<<256, 256, 0, s>>>(p.X, p.Y, (size_t)n * H);
      pf::rmsnorm<<<n, 256, 0, s>>>(p.X, mn, p.XN, H, p.eps, 1, 0);
      gemm(p.XN, reinterpret_cast<const uint16_t*>(p.arena + lo.gu), p.Y, n, 2 * F, H, 2 * F, s, p.blocked);
      pf::swiglu<<<n, 256, 0, s>>>(p.Y, p.HH, F);
      for (int k = 0; k < p.ndc; ++k) {  // W_down in chunk-major K chunks (one chunk when unsplit)
        const int k0 = k * p.kdc, kc = (F - k0) < p.kdc ? (F - k0) : p.kdc;
        gemm(p.HH + k0, reinterpret_cast<const uint16_t*>(p.arena + lo.d) + (size_t)H * k0, p.Y, n, H, kc, H, s, p.blocked, F, k);
      }
      pf::residual_add<<<256, 256, 0, s>>>(p.X, p.Y, (size_t)n * H);
    }
    if (!ck(cudaGetLastError(), "prefill chunk", err)) return MK_ERR_CUDA;
  }
  if (last_logits) {
    // final norm of each sequence's last token (row b * last_ct + last_ct - 1), then the LM head
    const uint16_t* fn = reinterpret_cast<const uint16_t*>(p.arena + p.off_fnorm);
    pf::rmsnorm<<<B, 256, 0, s>>>(p.X, fn, p.XN, H, p.eps, last_ct, last_ct - 1);
    gemm(p.XN, reinterpret_cast<const uint16_t*>(p.arena + p.off_lm), last_logits, B, p.V, H, p.V, s, p.blocked);
  }
  (void)last_t0;
  if (!ck(cudaGetLastError(), "prefill", err)) return MK_ERR_CUDA;
  return MK_OK;
}

}  // namespace mk
