// KDA recurrent decode step (Kimi K3 technical report, section 2.1.1 Eq. 1,
// applied to one token; section 5.4.2: the state is updated in place).
//
// Per (b, h):   a = exp(g)                     (per key channel i)
//               p_j = sum_i a_i k_i S_ij       (k^T of the decayed state)
//               r_j = sum_i a_i q_i S_ij       (q^T of the decayed state)
//               u_j = beta (v_j - p_j)
//               S_ij <- a_i S_ij + k_i u_j     (= (I - beta k k^T) Diag(a) S + beta k v^T)
//               o_j = scale (r_j + (q . k) u_j)   (= scale * S_new^T q)
//
// The step is HBM-bound (the fp32 state is read and written once; the token's
// q, k, v, g, beta are ~1 KB against 128 KB of state traffic per head at
// d = 128).  One CTA owns one (b, h): every thread loads its slice of S as
// float4 rows (a warp covers 128 contiguous floats = 512 B, fully coalesced),
// keeps it in registers, and all loads are issued before the first use so a
// CTA keeps 64 KB in flight.  Column sums over dk are reduced across the row
// groups through shared memory; the update is written back with float4
// stores.  Columns are independent, so no other cross-thread traffic exists.
#include <cuda_bf16.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <int DK, int DV>
struct DecodeShape {
  static constexpr int TPR = DV / 4;                             // threads per state row (float4 each)
  static constexpr int RP = (DK < 256 / TPR) ? DK : 256 / TPR;   // row groups
  static constexpr int NT = TPR * RP;                            // threads per CTA
  static constexpr int RPT = DK / RP;                            // rows per thread
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
    recurrent_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                          const TIn *__restrict__ v, const TIn *__restrict__ g,
                          const TIn *__restrict__ beta, float *S, TIn *__restrict__ o, float scale) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int TPR = Sh::TPR, RP = Sh::RP, NT = Sh::NT, RPT = Sh::RPT;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const int tx = tid % TPR, ty = tid / TPR;

  __shared__ float sk[DK], sq[DK], sa[DK], sv[DV];
  __shared__ float4 red_p[RP][TPR], red_r[RP][TPR];
  __shared__ float s_qk;

  // Issue every state load first: RPT float4 per thread, rows ty, ty+RP, ...
  float4 *S4 = reinterpret_cast<float4 *>(S + (size_t)bh * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = S4[(ty + r * RP) * TPR + tx];

  const size_t in_k = (size_t)bh * DK, in_v = (size_t)bh * DV;
  for (int i = tid; i < DK; i += NT) {
    sk[i] = to_f(k[in_k + i]);
    sq[i] = to_f(q[in_k + i]);
    sa[i] = expf(to_f(g[in_k + i]));
  }
  for (int j = tid; j < DV; j += NT) sv[j] = to_f(v[in_v + j]);
  const float b = to_f(beta[bh]);
  __syncthreads();

  if (tid < 32) {  // q . k, one warp
    float acc = 0.f;
    for (int i = tid; i < DK; i += 32) acc += sq[i] * sk[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (tid == 0) s_qk = acc;
  }

  float4 p = make_float4(0.f, 0.f, 0.f, 0.f), rr = p;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = ty + r * RP;
    const float a = sa[i], ka = sk[i], qa = sq[i];
    s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;  // decayed state, kept for the update
    p.x += ka * s[r].x; p.y += ka * s[r].y; p.z += ka * s[r].z; p.w += ka * s[r].w;
    rr.x += qa * s[r].x; rr.y += qa * s[r].y; rr.z += qa * s[r].z; rr.w += qa * s[r].w;
  }
  red_p[ty][tx] = p;
  red_r[ty][tx] = rr;
  __syncthreads();

  float4 P = red_p[0][tx];
#pragma unroll
  for (int y = 1; y < RP; ++y) {
    const float4 t = red_p[y][tx];
    P.x += t.x; P.y += t.y; P.z += t.z; P.w += t.w;
  }
  const int j0 = 4 * tx;
  float4 u;
  u.x = b * (sv[j0 + 0] - P.x);
  u.y = b * (sv[j0 + 1] - P.y);
  u.z = b * (sv[j0 + 2] - P.z);
  u.w = b * (sv[j0 + 3] - P.w);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = ty + r * RP;
    const float ki = sk[i];
    float4 t = s[r];
    t.x += ki * u.x; t.y += ki * u.y; t.z += ki * u.z; t.w += ki * u.w;
    S4[i * TPR + tx] = t;
  }
  if (ty == 0) {
    float4 R = red_r[0][tx];
#pragma unroll
    for (int y = 1; y < RP; ++y) {
      const float4 t = red_r[y][tx];
      R.x += t.x; R.y += t.y; R.z += t.z; R.w += t.w;
    }
    const float qk = s_qk;
    TIn *ob = o + in_v + j0;
    ob[0] = from_f<TIn>(scale * (R.x + qk * u.x));
    ob[1] = from_f<TIn>(scale * (R.y + qk * u.y));
    ob[2] = from_f<TIn>(scale * (R.z + qk * u.z));
    ob[3] = from_f<TIn>(scale * (R.w + qk * u.w));
  }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t st) {
  const int n = a.B * a.H;
  recurrent_step_kernel<DK, DV, TIn><<<n, DecodeShape<DK, DV>::NT, 0, st>>>(
      (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.g,
      (const TIn *)a.beta, a.S, (TIn *)a.o, a.scale);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_dt(const DecodeArgs &a, cudaStream_t st) {
#define KDA_DEC_CASE(DKv, DVv) \
  if (a.dk == DKv && a.dv == DVv) return launch_t<DKv, DVv, TIn>(a, st);
#define KDA_DEC_ROW(DKv) KDA_DEC_CASE(DKv, 16) KDA_DEC_CASE(DKv, 32) KDA_DEC_CASE(DKv, 64) KDA_DEC_CASE(DKv, 128)
  KDA_DEC_ROW(16) KDA_DEC_ROW(32) KDA_DEC_ROW(64) KDA_DEC_ROW(128)
#undef KDA_DEC_ROW
#undef KDA_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent_step(const DecodeArgs &a, cudaStream_t st) {
  if (a.B * a.H == 0) return cudaSuccess;
  return a.bf16 ? launch_dt<__nv_bfloat16>(a, st) : launch_dt<float>(a, st);
}

}  // namespace kda
