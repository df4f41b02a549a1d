// Output edge of a KDA layer (Kimi K3 report, section 2.1.1, Eq. 6): the
// recurrent output o of each head is normalised by a per-head RMSNorm and
// multiplied by a data-dependent sigmoid gate,
//     y[b,h,t,:] = Sigmoid(gate[b,h,t,:]) * w[h,:] * o[b,h,t,:] / sqrt(mean_j o[b,h,t,j]^2 + eps)
// (W_g x and W_o of Eq. 6 are dense projections outside this kernel: `gate`
// is W_g x already split into heads).
//
// HBM-bound: every (b, h, t) row of dv values is read twice (o, gate) and
// written once.  One warp owns one row: lane l holds columns l, l + 32, ...
// (dv = 128 in bf16: four consecutive values, one 8-byte load per tensor),
// the sum of squares is a warp shuffle reduction, all arithmetic is fp32 and
// y is rounded to the input dtype (RNE).  8 rows per 256-thread CTA.
#include <cuda_bf16.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kRowsPerCta = 8;

__device__ __forceinline__ float ld(const float *p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float *p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + __expf(-x)); }

// Generic rows: any dv that is a multiple of 16 up to 128, either dtype.
template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerCta)
    out_gate_kernel(const T *__restrict__ o, const T *__restrict__ gate, const float *__restrict__ w,
                    T *__restrict__ y, long long rows, int H, int T_len, int dv, float eps) {
  const long long row = (long long)blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = (int)((row / T_len) % H);
  const T *orow = o + row * dv;
  const T *grow = gate + row * dv;
  float ov[4], ss = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = lane + 32 * u;
    ov[u] = j < dv ? ld(orow + j) : 0.f;
    ss += ov[u] * ov[u];
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  const float inv = rsqrtf(ss / (float)dv + eps);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = lane + 32 * u;
    if (j < dv) st(y + row * dv + j, sigmoid(ld(grow + j)) * w[h * dv + j] * ov[u] * inv);
  }
}

// bf16 rows of 128: lane l holds columns 4l .. 4l + 3 (one 8-byte load per tensor).
// (Four rows per warp with all loads issued first measured slower here: fewer
// CTAs for a launch this short.)
__global__ void __launch_bounds__(32 * kRowsPerCta)
    out_gate_bf16_128_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ gate,
                             const float *__restrict__ w, __nv_bfloat16 *__restrict__ y, long long rows, int H,
                             int T_len, float eps) {
  const long long row = (long long)blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = (int)((row / T_len) % H);
  const uint2 ob = __ldg(reinterpret_cast<const uint2 *>(o + row * 128) + lane);
  const uint2 gb = __ldg(reinterpret_cast<const uint2 *>(gate + row * 128) + lane);
  const float4 wv = __ldg(reinterpret_cast<const float4 *>(w + h * 128) + lane);
  const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ob.x));
  const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ob.y));
  const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gb.x));
  const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gb.y));
  float ss = o01.x * o01.x + o01.y * o01.y + o23.x * o23.x + o23.y * o23.y;
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  const float inv = rsqrtf(ss * (1.f / 128.f) + eps);
  const __nv_bfloat162 y01 =
      __floats2bfloat162_rn(sigmoid(g01.x) * wv.x * o01.x * inv, sigmoid(g01.y) * wv.y * o01.y * inv);
  const __nv_bfloat162 y23 =
      __floats2bfloat162_rn(sigmoid(g23.x) * wv.z * o23.x * inv, sigmoid(g23.y) * wv.w * o23.y * inv);
  uint2 yb;
  yb.x = *reinterpret_cast<const uint32_t *>(&y01);
  yb.y = *reinterpret_cast<const uint32_t *>(&y23);
  reinterpret_cast<uint2 *>(y + row * 128)[lane] = yb;
}

}  // namespace

cudaError_t launch_out_gate(const OutGateArgs &a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.H * a.T;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta);
  if (a.bf16 && a.dv == 128)
    out_gate_bf16_128_kernel<<<blocks, 32 * kRowsPerCta, 0, st>>>(
        (const __nv_bfloat16 *)a.o, (const __nv_bfloat16 *)a.gate, a.w, (__nv_bfloat16 *)a.y, rows, a.H, a.T, a.eps);
  else if (a.bf16)
    out_gate_kernel<__nv_bfloat16><<<blocks, 32 * kRowsPerCta, 0, st>>>(
        (const __nv_bfloat16 *)a.o, (const __nv_bfloat16 *)a.gate, a.w, (__nv_bfloat16 *)a.y, rows, a.H, a.T, a.dv,
        a.eps);
  else
    out_gate_kernel<float><<<blocks, 32 * kRowsPerCta, 0, st>>>((const float *)a.o, (const float *)a.gate, a.w,
                                                                (float *)a.y, rows, a.H, a.T, a.dv, a.eps);
  return cudaGetLastError();
}

}  // namespace kda
