// Speculative-decode replay and verify (Kimi K3 report, section 5.4.2).
//
// With MTP speculative decoding the verifier may reject part of the draft,
// and an in-place state cannot be rolled back.  The report caches only the
// projected inputs of the draft tokens (far smaller than the state), rebuilds
// the state of the accepted ones on chip, and runs the replayed tokens and the
// next window through one recurrent loop in one kernel.  Here, per (b, h), one
// CTA loads the committed state S once, then for the W tokens of the window:
//   tokens t <  n_replay[b]  (accepted drafts, cached inputs): advance S;
//                            after the last one S is written back (committed);
//   tokens t >= n_replay[b]  (bonus token and next draft): advance S on chip
//                            and write o_t for verification; never committed.
// Each token is the decode step of Eq. 1 (same thread layout as the decode
// kernel: rows of S in registers as float4, column sums over dk reduced
// through shared memory), so the window costs one read and at most one write
// of the state instead of one of each per token.
#include <cuda_bf16.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void put(float *p, float x) { *p = x; }
__device__ __forceinline__ void put(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int DK, int DV>
struct SpecShape {
  static constexpr int TPR = DV / 4;                             // threads per state row (float4 each)
  static constexpr int RP = (DK < 256 / TPR) ? DK : 256 / TPR;   // row groups
  static constexpr int NT = TPR * RP;                            // threads per CTA
  static constexpr int RPT = DK / RP;                            // rows per thread
};

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(SpecShape<DK, DV>::NT)
    spec_replay_verify_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                              const TIn *__restrict__ g, const TIn *__restrict__ beta, float *S,
                              TIn *__restrict__ o, const int *__restrict__ n_replay, int H, int W, float scale) {
  using Sh = SpecShape<DK, DV>;
  constexpr int TPR = Sh::TPR, RP = Sh::RP, NT = Sh::NT, RPT = Sh::RPT;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const int tx = tid % TPR, ty = tid / TPR;
  __shared__ float sk[DK], sq[DK], sa[DK], sv[DV];
  __shared__ float4 red_p[RP][TPR], red_r[RP][TPR];
  __shared__ float s_qk, s_b;

  const int nr = min(max(n_replay[bh / H], 0), W);
  float4 *S4 = reinterpret_cast<float4 *>(S + (size_t)bh * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = S4[(ty + r * RP) * TPR + tx];

  for (int t = 0; t < W; ++t) {
    const size_t in_k = ((size_t)bh * W + t) * DK, in_v = ((size_t)bh * W + t) * DV;
    for (int i = tid; i < DK; i += NT) {
      sk[i] = to_f(k[in_k + i]);
      sq[i] = to_f(q[in_k + i]);
      sa[i] = expf(to_f(g[in_k + i]));
    }
    for (int j = tid; j < DV; j += NT) sv[j] = to_f(v[in_v + j]);
    if (tid == 0) s_b = to_f(beta[(size_t)bh * W + t]);
    __syncthreads();
    const bool out = t >= nr;
    if (out && tid < 32) {  // q . k, one warp
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
      s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
      p.x += ka * s[r].x; p.y += ka * s[r].y; p.z += ka * s[r].z; p.w += ka * s[r].w;
      rr.x += qa * s[r].x; rr.y += qa * s[r].y; rr.z += qa * s[r].z; rr.w += qa * s[r].w;
    }
    red_p[ty][tx] = p;
    red_r[ty][tx] = rr;
    __syncthreads();
    float4 P = red_p[0][tx];
#pragma unroll
    for (int y = 1; y < RP; ++y) {
      const float4 c = red_p[y][tx];
      P.x += c.x; P.y += c.y; P.z += c.z; P.w += c.w;
    }
    const int j0 = 4 * tx;
    const float b = s_b;
    const float4 u = make_float4(b * (sv[j0 + 0] - P.x), b * (sv[j0 + 1] - P.y), b * (sv[j0 + 2] - P.z),
                                 b * (sv[j0 + 3] - P.w));
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float ki = sk[ty + r * RP];
      s[r].x += ki * u.x; s[r].y += ki * u.y; s[r].z += ki * u.z; s[r].w += ki * u.w;
    }
    if (t == nr - 1)  // the last accepted token: this state is committed
#pragma unroll
      for (int r = 0; r < RPT; ++r) S4[(ty + r * RP) * TPR + tx] = s[r];
    if (out && ty == 0) {
      float4 R = red_r[0][tx];
#pragma unroll
      for (int y = 1; y < RP; ++y) {
        const float4 c = red_r[y][tx];
        R.x += c.x; R.y += c.y; R.z += c.z; R.w += c.w;
      }
      const float qk = s_qk;
      TIn *ob = o + in_v + j0;
      put(ob + 0, scale * (R.x + qk * u.x));
      put(ob + 1, scale * (R.y + qk * u.y));
      put(ob + 2, scale * (R.z + qk * u.z));
      put(ob + 3, scale * (R.w + qk * u.w));
    }
    __syncthreads();  // this token's shared inputs and partial sums are consumed
  }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_t(const SpecArgs &a, cudaStream_t st) {
  spec_replay_verify_kernel<DK, DV, TIn><<<a.B * a.H, SpecShape<DK, DV>::NT, 0, st>>>(
      (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.g, (const TIn *)a.beta, a.S,
      (TIn *)a.o, a.n_replay, a.H, a.W, a.scale);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_dt(const SpecArgs &a, cudaStream_t st) {
#define KDA_SP_CASE(DKv, DVv) \
  if (a.dk == DKv && a.dv == DVv) return launch_t<DKv, DVv, TIn>(a, st);
#define KDA_SP_ROW(DKv) KDA_SP_CASE(DKv, 16) KDA_SP_CASE(DKv, 32) KDA_SP_CASE(DKv, 64) KDA_SP_CASE(DKv, 128)
  KDA_SP_ROW(16) KDA_SP_ROW(32) KDA_SP_ROW(64) KDA_SP_ROW(128)
#undef KDA_SP_ROW
#undef KDA_SP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_spec_replay_verify(const SpecArgs &a, cudaStream_t st) {
  if (a.B * a.H == 0 || a.W == 0) return cudaSuccess;
  return a.bf16 ? launch_dt<__nv_bfloat16>(a, st) : launch_dt<float>(a, st);
}

}  // namespace kda
