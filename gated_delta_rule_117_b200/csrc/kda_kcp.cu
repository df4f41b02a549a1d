// Cross-device KDA context parallelism, prefix step (Kimi K3 report,
// section 5.1.2, Eq. 17).  A segment maps its entering state S to S~ + M S,
// so once every rank has the (M_r, S~_r) of all earlier segments (one
// all-gather), the state entering rank R's segment is the composition
//     S_in = M_{R-1} (... (M_0 h0 + S~_0) ...) + S~_{R-1},
// computed here in fp32 on the device.  Grid (B*H, dv/16): each CTA carries 16
// state columns of one chain through the R steps; M_r is staged in shared
// memory with a padded row (conflict-free reads of M[i][k] by consecutive i).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kCols = 16;

__global__ void __launch_bounds__(256) kcp_compose_kernel(const float *M, const float *St, const float *h0,
                                                          float *S_in, int R, int BH, int dk, int dv) {
  extern __shared__ float sm[];
  float *Ms = sm;                      // [dk][dk + 1]
  float *X = sm + dk * (dk + 1);       // [dk][kCols]
  const int bh = blockIdx.x, c0 = kCols * blockIdx.y, tid = threadIdx.x;
  const int i = tid >> 1, j0 = 8 * (tid & 1);  // row i, columns j0 .. j0 + 7 of the CTA's 16
  const bool active = i < dk;
  const size_t sdv = (size_t)dk * dv, sdk = (size_t)dk * dk;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    acc[j] = (active && h0) ? h0[bh * sdv + (size_t)i * dv + c0 + j0 + j] : 0.f;
  for (int r = 0; r < R; ++r) {
    if (active)
#pragma unroll
      for (int j = 0; j < 8; ++j) X[i * kCols + j0 + j] = acc[j];
    const float *Mg = M + ((size_t)r * BH + bh) * sdk;
    for (int e = tid; e < dk * dk; e += 256) Ms[(e / dk) * (dk + 1) + e % dk] = Mg[e];
    __syncthreads();
    if (active) {
      const float *Sg = St + ((size_t)r * BH + bh) * sdv + (size_t)i * dv + c0 + j0;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = Sg[j];
      for (int k = 0; k < dk; ++k) {
        const float m = Ms[i * (dk + 1) + k];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += m * X[k * kCols + j0 + j];
      }
    }
    __syncthreads();
  }
  if (active)
#pragma unroll
    for (int j = 0; j < 8; ++j) S_in[bh * sdv + (size_t)i * dv + c0 + j0 + j] = acc[j];
}

}  // namespace

cudaError_t launch_kcp_compose(const float *M, const float *St, const float *h0, float *S_in, int R, int BH, int dk,
                               int dv, cudaStream_t st) {
  if (BH == 0) return cudaSuccess;
  const int smem = (dk * (dk + 1) + dk * kCols) * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kcp_compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kcp_compose_kernel<<<dim3(BH, dv / kCols), 256, smem, st>>>(M, St, h0, S_in, R, BH, dk, dv);
  return cudaGetLastError();
}

}  // namespace kda
