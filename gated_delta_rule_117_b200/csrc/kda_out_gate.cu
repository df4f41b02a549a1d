// Output edge of a KDA layer (Kimi K3 report, section 2.1.1, Eq. 6): the
// recurrent output o of each head is normalised by a per-head RMSNorm and
// multiplied by a data-dependent sigmoid gate,
//     y[b,h,t,:] = Sigmoid(gate[b,h,t,:]) * w[h,:] * o[b,h,t,:] / sqrt(mean_j o[b,h,t,j]^2 + eps)
// (W_g x and W_o of Eq. 6 are dense projections outside this kernel: `gate`
// is W_g x already split into heads).
//
// HBM-bound: every (b, h, t) row of dv values is read twice (o, gate) and
// written once.  Generic rows: one warp owns one row, lane l holds columns l,
// l + 32, ...; bf16 rows of 128: half a warp per row (below).  The sum of
// squares is a shuffle reduction, all arithmetic is fp32 and y is rounded to
// the input dtype (RNE).
#include <cuda_bf16.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kRowsPerCta = 8;

__device__ __forceinline__ float ld(const float *p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float *p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// fast reciprocal division (the Eq. 6 gate of the fused paths uses the same form):
// an IEEE division here made the pass instruction-bound
__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

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

// bf16 rows of 128: half a warp per row, lane l holding columns 8(l & 15) ..
// 8(l & 15) + 7 (one 16-byte load per tensor), two rows per warp.  Measured on
// the 2^24-row edge of the long workload: 0.72 of the copy bandwidth, against
// 0.58 for one row per warp with 8-byte loads, 0.66 / 0.45 for four / eight
// rows per warp (more registers, fewer resident warps), and 0.51 for a
// pipeline of bulk copies into shared memory.
constexpr int kRowsPerWarp = 2;

__device__ __forceinline__ float2 bf2(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
}
__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(32 * kRowsPerCta)
    out_gate_bf16_128_kernel(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ gate,
                             const float *__restrict__ w, __nv_bfloat16 *__restrict__ y, long long rows, int H,
                             int T_len, float eps) {
  constexpr int kIt = kRowsPerWarp / 2;  // two rows (one per half-warp) per step
  const long long row0 = ((long long)blockIdx.x * kRowsPerCta + (threadIdx.x >> 5)) * kRowsPerWarp;
  const int lane = threadIdx.x & 31, half = lane >> 4, col = lane & 15;
  uint4 ob[kIt], gb[kIt];
#pragma unroll
  for (int i = 0; i < kIt; ++i) {
    const long long row = row0 + 2 * i + half;
    if (row < rows) {
      ob[i] = __ldg(reinterpret_cast<const uint4 *>(o + row * 128) + col);
      gb[i] = __ldg(reinterpret_cast<const uint4 *>(gate + row * 128) + col);
    } else {
      ob[i] = gb[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int i = 0; i < kIt; ++i) {
    const long long row = row0 + 2 * i + half;
    const uint32_t ow[4] = {ob[i].x, ob[i].y, ob[i].z, ob[i].w};
    const uint32_t gw[4] = {gb[i].x, gb[i].y, gb[i].z, gb[i].w};
    float2 ov[4];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ov[u] = bf2(ow[u]);
      ss += ov[u].x * ov[u].x + ov[u].y * ov[u].y;
    }
    // the 16 lanes of this half-warp hold the row (the xor masks stay inside it);
    // all 32 lanes take part, rows past the end with zeros
#pragma unroll
    for (int m = 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if (row >= rows) continue;
    const float inv = rsqrtf(ss * (1.f / 128.f) + eps);
    const int h = (int)((row / T_len) % H);
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(w + h * 128) + 2 * col);
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(w + h * 128) + 2 * col + 1);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    uint32_t yw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 g = bf2(gw[u]);
      yw[u] = pack_bf2(sigmoid(g.x) * wv[2 * u] * ov[u].x * inv, sigmoid(g.y) * wv[2 * u + 1] * ov[u].y * inv);
    }
    reinterpret_cast<uint4 *>(y + row * 128)[col] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
  }
}

}  // namespace

cudaError_t launch_out_gate(const OutGateArgs &a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.H * a.T;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta);
  const long long rows_per_cta128 = (long long)kRowsPerCta * kRowsPerWarp;
  if (a.bf16 && a.dv == 128)
    out_gate_bf16_128_kernel<<<(unsigned)((rows + rows_per_cta128 - 1) / rows_per_cta128), 32 * kRowsPerCta, 0, st>>>(
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
