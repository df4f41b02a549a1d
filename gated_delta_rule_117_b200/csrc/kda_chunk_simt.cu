// KDA chunked prefill on CUDA cores, fp32 arithmetic, 16-token chunks.
//
// Chunkwise-parallel form of the Kimi K3 technical report (section 2.1.1,
// Eq. 3 cumulative decay, Eq. 4 outputs, UT transform).  For a chunk of C = 16
// tokens with entering state S and chunk-local inclusive log-decay
// G_r = sum_{s<=r} g_s (a 16-token window stays in [-80, 0] under the report's
// lower-bounded gate, so e^{+-G} is finite in fp32):
//
//   A  = Tril_incl[(Q e^G)(K e^-G)^T]          L = StrictTril[Diag(beta)(K e^G)(K e^-G)^T]
//   T  = (I + L)^-1 Diag(beta)                 (forward substitution, fp32)
//   U  = T V,  W = T (K e^G),  V~ = U - W S     (pseudo-values)
//   O  = scale [(Q e^G) S + A V~]
//   S' = Diag(e^{G_C}) S + (K e^{G_C - G})^T V~
//
// One CTA (256 threads) carries one (b, h) chain through all its chunks with
// S resident in shared memory.  A ragged last chunk is zero padded (g = 0 keeps
// the cumulative decay flat, beta = 0 removes the padded rows).  This kernel is
// the fp32 path and the portable fallback for every supported d; the bf16
// d = 128 workloads use the tensor-core kernel.
#include <cuda_bf16.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = 16;
constexpr int NT = 256;

template <typename T>
__device__ __forceinline__ float ld_f(const T *p);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ void st_f(float *p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int DK, int DV>
struct SimtSmem {
  static constexpr int LK = DK + 1;  // padded row stride of [C][DK] tiles (column reads)
  static constexpr int oS = 0;                 // S   [DK][DV]
  static constexpr int oQe = oS + DK * DV;     // Q e^G        [C][LK]
  static constexpr int oKn = oQe + C * LK;     // K e^-G       [C][LK]
  static constexpr int oKe = oKn + C * LK;     // K e^G        [C][LK]
  static constexpr int oKc = oKe + C * LK;     // K e^(G_C-G)  [C][LK]
  static constexpr int oW = oKc + C * LK;      // W            [C][LK]
  static constexpr int oV = oW + C * LK;       // V, then V~   [C][DV]
  static constexpr int oU = oV + C * DV;       // U            [C][DV]
  static constexpr int oA = oU + C * DV;       // A            [C][C+1]
  static constexpr int oL = oA + C * (C + 1);  // L            [C][C+1]
  static constexpr int oT = oL + C * (C + 1);  // T            [C][C+1]
  static constexpr int oB = oT + C * (C + 1);  // beta         [C]
  static constexpr int oGC = oB + C;           // e^{G_C}      [DK]
  static constexpr int total = oGC + DK;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(NT, 1)
    chunk16_kernel(const TIn *__restrict__ qg, const TIn *__restrict__ kg, const TIn *__restrict__ vg,
                   const TIn *__restrict__ gg, const TIn *__restrict__ betag,
                   const float *h0, TIn *__restrict__ og, float *hT, int T, float scale, float *ckpt,
                   int ckpt_interval, int n_ckpt, const float *A_log, float g_min, int H) {
  using L = SimtSmem<DK, DV>;
  constexpr int LK = L::LK;
  constexpr int CPT = DV / 16;  // output columns per thread in (row, column-group) layouts
  extern __shared__ float sm[];
  float *S = sm + L::oS, *Qe = sm + L::oQe, *Kn = sm + L::oKn, *Ke = sm + L::oKe, *Kc = sm + L::oKc;
  float *Wm = sm + L::oW, *Vs = sm + L::oV, *Us = sm + L::oU, *Am = sm + L::oA, *Lm = sm + L::oL;
  float *Tm = sm + L::oT, *bet = sm + L::oB, *gC = sm + L::oGC;

  const int tid = threadIdx.x;
  const size_t bh = blockIdx.x;
  const TIn *q = qg + bh * (size_t)T * DK, *k = kg + bh * (size_t)T * DK, *g = gg + bh * (size_t)T * DK;
  const TIn *v = vg + bh * (size_t)T * DV, *beta = betag + bh * (size_t)T;
  TIn *o = og + bh * (size_t)T * DV;

  for (int e = tid; e < DK * DV; e += NT) S[e] = h0 ? h0[bh * DK * DV + e] : 0.f;

  // (row, column-group) thread layout for [C][DV] outputs: row r = tid / 16,
  // columns jg + 16 u (consecutive threads -> consecutive columns).
  const int rr = tid / 16, jg = tid % 16;

  for (int t0 = 0; t0 < T; t0 += C) {
    const int n = min(C, T - t0);
    __syncthreads();  // previous chunk's state update is complete
    // ---- load the chunk (zero padded) -------------------------------------
    for (int e = tid; e < C * DK; e += NT) {
      const int r = e / DK, c = e % DK;
      const bool ok = r < n;
      const size_t off = (size_t)(t0 + r) * DK + c;
      Qe[r * LK + c] = ok ? ld_f(q + off) : 0.f;
      Kn[r * LK + c] = ok ? ld_f(k + off) : 0.f;
      float gv = ok ? ld_f(g + off) : 0.f;  // raw g for the cumsum
      if (A_log && ok)  // fused Eq. 5 gate: the input holds the logits z
        gv = g_min / (1.f + expf(-expf(A_log[(bh % H) * DK + c]) * gv));
      Kc[r * LK + c] = gv;
    }
    for (int e = tid; e < C * DV; e += NT) {
      const int r = e / DV, c = e % DV;
      Vs[e] = r < n ? ld_f(v + (size_t)(t0 + r) * DV + c) : 0.f;
    }
    if (tid < C) bet[tid] = tid < n ? ld_f(beta + t0 + tid) : 0.f;
    __syncthreads();
    // ---- a-1: chunk-local inclusive cumulative log-decay and its factors ----
    if (tid < DK) {
      const int c = tid;
      float G = 0.f;
      for (int r = 0; r < C; ++r) {
        G += Kc[r * LK + c];
        Kc[r * LK + c] = G;  // store G_r
      }
      const float GC = G;
      gC[c] = expf(GC);
      for (int r = 0; r < C; ++r) {
        const float Gr = Kc[r * LK + c];
        const float kr = Kn[r * LK + c];
        const float e = expf(Gr);
        Qe[r * LK + c] *= e;
        Ke[r * LK + c] = kr * e;
        Kn[r * LK + c] = kr * expf(-Gr);
        Kc[r * LK + c] = kr * expf(GC - Gr);
      }
    }
    __syncthreads();
    // ---- a-2: decayed intra-chunk Gram matrices A and L ---------------------
    {
      const int r = tid / C, j = tid % C;
      float a = 0.f, l = 0.f;
      if (j <= r) {
        for (int c = 0; c < DK; ++c) {
          const float kn = Kn[j * LK + c];
          a += Qe[r * LK + c] * kn;
          l += Ke[r * LK + c] * kn;
        }
      }
      Am[r * (C + 1) + j] = j <= r ? a : 0.f;
      Lm[r * (C + 1) + j] = j < r ? bet[r] * l : 0.f;
    }
    __syncthreads();
    // ---- a-3: T = (I + L)^-1 Diag(beta), one column per thread -------------
    if (tid < C) {
      const int j = tid;
      float x[C];
#pragma unroll
      for (int r = 0; r < C; ++r) {
        float acc = (r == j) ? bet[j] : 0.f;
#pragma unroll
        for (int s = 0; s < r; ++s) acc -= Lm[r * (C + 1) + s] * x[s];
        x[r] = acc;
        Tm[r * (C + 1) + j] = acc;
      }
    }
    __syncthreads();
    // ---- a-3: U = T V, W = T (K e^G) ----------------------------------------
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
      const int j = jg + 16 * u;
      float acc = 0.f;
      for (int s = 0; s <= rr; ++s) acc += Tm[rr * (C + 1) + s] * Vs[s * DV + j];
      Us[rr * DV + j] = acc;
    }
    for (int e = tid; e < C * DK; e += NT) {
      const int r = e / DK, c = e % DK;
      float acc = 0.f;
      for (int s = 0; s <= r; ++s) acc += Tm[r * (C + 1) + s] * Ke[s * LK + c];
      Wm[r * LK + c] = acc;
    }
    __syncthreads();
    // ---- a-4: V~ = U - W S and the inter-chunk part (Q e^G) S ---------------
    float oacc[CPT];
    {
      float vt[CPT];
#pragma unroll
      for (int u = 0; u < CPT; ++u) { vt[u] = 0.f; oacc[u] = 0.f; }
      for (int c = 0; c < DK; ++c) {
        const float w = Wm[rr * LK + c], qe = Qe[rr * LK + c];
#pragma unroll
        for (int u = 0; u < CPT; ++u) {
          const float sv = S[c * DV + jg + 16 * u];
          vt[u] += w * sv;
          oacc[u] += qe * sv;
        }
      }
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        const int j = jg + 16 * u;
        Vs[rr * DV + j] = Us[rr * DV + j] - vt[u];  // V~ replaces V
      }
    }
    __syncthreads();
    // ---- a-4/a-6: O = scale [(Q e^G) S + A V~] ------------------------------
    if (rr < n) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        const int j = jg + 16 * u;
        float acc = oacc[u];
        for (int s = 0; s <= rr; ++s) acc += Am[rr * (C + 1) + s] * Vs[s * DV + j];
        st_f(o + (size_t)(t0 + rr) * DV + j, scale * acc);
      }
    }
    // ---- a-4: S' = Diag(e^{G_C}) S + (K e^{G_C-G})^T V~ ----------------------
    for (int e = tid; e < DK * DV; e += NT) {
      const int i = e / DV, j = e % DV;
      float acc = gC[i] * S[e];
#pragma unroll
      for (int r = 0; r < C; ++r) acc += Kc[r * LK + i] * Vs[r * DV + j];
      S[e] = acc;
    }
    // state checkpoint at a hash-aligned position (prefix caching)
    const int pend = t0 + C;
    if (ckpt && pend <= T && pend % ckpt_interval == 0) {
      __syncthreads();
      float *dst = ckpt + (bh * n_ckpt + pend / ckpt_interval - 1) * (size_t)(DK * DV);
      for (int e = tid; e < DK * DV; e += NT) dst[e] = S[e];
    }
  }
  __syncthreads();
  if (hT)
    for (int e = tid; e < DK * DV; e += NT) hT[bh * DK * DV + e] = S[e];
}

template <int DK, int DV, typename TIn>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t st) {
  constexpr size_t smem = SimtSmem<DK, DV>::bytes;
  auto kern = chunk16_kernel<DK, DV, TIn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.B * a.H, NT, smem, st>>>((const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v,
                                    (const TIn *)a.g, (const TIn *)a.beta, a.h0, (TIn *)a.o, a.hT,
                                    a.T, a.scale, a.ckpt, a.ckpt_interval, a.n_ckpt, a.A_log, a.g_min, a.H);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_dt(const ChunkArgs &a, cudaStream_t st) {
#define KDA_CH_CASE(DKv, DVv) \
  if (a.dk == DKv && a.dv == DVv) return launch_t<DKv, DVv, TIn>(a, st);
#define KDA_CH_ROW(DKv) KDA_CH_CASE(DKv, 16) KDA_CH_CASE(DKv, 32) KDA_CH_CASE(DKv, 64) KDA_CH_CASE(DKv, 128)
  KDA_CH_ROW(16) KDA_CH_ROW(32) KDA_CH_ROW(64) KDA_CH_ROW(128)
#undef KDA_CH_ROW
#undef KDA_CH_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_simt16(const ChunkArgs &a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return a.bf16 ? launch_dt<__nv_bfloat16>(a, st) : launch_dt<float>(a, st);
}

}  // namespace kda
