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
// of the state instead of one of each per token.  The window's inputs are
// staged in shared memory once (in blocks of WB tokens) while the state load
// is in flight; the column partial sums are double-buffered by token parity,
// so each token costs one barrier; the q-side sums are formed only for the
// tokens whose output is verified.  For dk = dv = 128 a warp-sliced variant
// (below) replaces the per-token barrier with shuffles inside each warp.
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
  static constexpr int WB = 8;                                   // window tokens staged at a time
};

__device__ __forceinline__ float2 lo2(float4 a) { return make_float2(a.x, a.y); }
__device__ __forceinline__ float2 hi2(float4 a) { return make_float2(a.z, a.w); }

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(SpecShape<DK, DV>::NT)
    spec_replay_verify_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                              const TIn *__restrict__ g, const TIn *__restrict__ beta, float *S,
                              TIn *__restrict__ o, const int *__restrict__ n_replay, int H, int W, float scale) {
  using Sh = SpecShape<DK, DV>;
  constexpr int TPR = Sh::TPR, RP = Sh::RP, NT = Sh::NT, RPT = Sh::RPT, WB = Sh::WB;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const int tx = tid % TPR, ty = tid / TPR;
  // a block of up to WB window tokens, staged once: k, q, alpha = exp(g), v, beta, q.k
  __shared__ float sk[WB][DK], sq[WB][DK], sa[WB][DK], sv[WB][DV], sb[WB], sqk[WB];
  // column partial sums, double-buffered by token parity: one barrier per token
  __shared__ float4 red_p[2][RP][TPR], red_r[2][RP][TPR];

  const int nr = min(max(n_replay[bh / H], 0), W);
  float4 *S4 = reinterpret_cast<float4 *>(S + (size_t)bh * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = S4[(ty + r * RP) * TPR + tx];  // in flight while the window is staged

  for (int t0 = 0; t0 < W; t0 += WB) {
    const int nb = min(WB, W - t0);
    if (t0 > 0) __syncthreads();  // the previous block's staged inputs are consumed
    for (int e = tid; e < nb * DK; e += NT) {
      const int u = e / DK, i = e % DK;
      const size_t in = ((size_t)bh * W + t0 + u) * DK + i;
      sk[u][i] = to_f(k[in]);
      sq[u][i] = to_f(q[in]);
      sa[u][i] = expf(to_f(g[in]));
    }
    for (int e = tid; e < nb * DV; e += NT) {
      const int u = e / DV, j = e % DV;
      sv[u][j] = to_f(v[((size_t)bh * W + t0 + u) * DV + j]);
    }
    if (tid < nb) sb[tid] = to_f(beta[(size_t)bh * W + t0 + tid]);
    __syncthreads();
    // q . k of each staged token: one warp per token
    for (int u = tid >> 5; u < nb; u += NT / 32) {
      float acc = 0.f;
      for (int i = tid & 31; i < DK; i += 32) acc += sq[u][i] * sk[u][i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if ((tid & 31) == 0) sqk[u] = acc;
    }
    // (sqk is read after the first token's barrier below)
    for (int u = 0; u < nb; ++u) {
      const int t = t0 + u, par = t & 1;
      const bool out = t >= nr;  // bonus / draft token: its output is verified
      float2 p0 = make_float2(0.f, 0.f), p1 = p0, r0 = p0, r1 = p0;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = ty + r * RP;
        const float2 a = make_float2(sa[u][i], sa[u][i]), ka = make_float2(sk[u][i], sk[u][i]);
        float2 x0 = __fmul2_rn(a, lo2(s[r])), x1 = __fmul2_rn(a, hi2(s[r]));
        s[r] = make_float4(x0.x, x0.y, x1.x, x1.y);
        p0 = __ffma2_rn(ka, x0, p0);
        p1 = __ffma2_rn(ka, x1, p1);
        if (out) {
          const float2 qa = make_float2(sq[u][i], sq[u][i]);
          r0 = __ffma2_rn(qa, x0, r0);
          r1 = __ffma2_rn(qa, x1, r1);
        }
      }
      red_p[par][ty][tx] = make_float4(p0.x, p0.y, p1.x, p1.y);
      if (out) red_r[par][ty][tx] = make_float4(r0.x, r0.y, r1.x, r1.y);
      __syncthreads();
      float4 P = red_p[par][0][tx];
#pragma unroll
      for (int y = 1; y < RP; ++y) {
        const float4 c = red_p[par][y][tx];
        P.x += c.x; P.y += c.y; P.z += c.z; P.w += c.w;
      }
      const int j0 = 4 * tx;
      const float b = sb[u];
      const float4 vj = *reinterpret_cast<const float4 *>(&sv[u][j0]);
      const float4 uu = make_float4(b * (vj.x - P.x), b * (vj.y - P.y), b * (vj.z - P.z), b * (vj.w - P.w));
      const float2 u0 = lo2(uu), u1 = hi2(uu);
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float2 ki = make_float2(sk[u][ty + r * RP], sk[u][ty + r * RP]);
        const float2 x0 = __ffma2_rn(ki, u0, lo2(s[r])), x1 = __ffma2_rn(ki, u1, hi2(s[r]));
        s[r] = make_float4(x0.x, x0.y, x1.x, x1.y);
      }
      if (t == nr - 1)  // the last accepted token: this state is committed
#pragma unroll
        for (int r = 0; r < RPT; ++r) S4[(ty + r * RP) * TPR + tx] = s[r];
      if (out && ty == 0) {
        float4 R = red_r[par][0][tx];
#pragma unroll
        for (int y = 1; y < RP; ++y) {
          const float4 c = red_r[par][y][tx];
          R.x += c.x; R.y += c.y; R.z += c.z; R.w += c.w;
        }
        const float qk = sqk[u];
        TIn *ob = o + ((size_t)bh * W + t) * DV + j0;
        put(ob + 0, scale * (R.x + qk * uu.x));
        put(ob + 1, scale * (R.y + qk * uu.y));
        put(ob + 2, scale * (R.z + qk * uu.z));
        put(ob + 3, scale * (R.w + qk * uu.w));
      }
      // red_*[par] is rewritten two tokens later, after the next token's barrier
    }
  }
}

// dk = dv = 128: a warp owns a 16-column slice of the state over all 128 rows
// (lane = row group rg = lane / 4 of 8, column group cg = lane % 4 of 4 float4
// columns; rows rg, rg + 8, ..., rg + 120 in registers), so the column sums
// over dk finish with three butterfly shuffles inside the warp and a token
// needs no barrier: the warps of a CTA run through the window independently.
constexpr int kD = 128, kWarps = 8, kRowsPT = 16, kWB = 8;

// kFused: the same loop with the KDA layer's gate edges folded in, as the
// report's replay kernel does (section 5.4.2): g arrives as the Eq. 5 logits z
// (g = g_min Sigmoid(e^A z), formed while the window is staged) and the
// verified outputs leave as the Eq. 6 edge y = Sigmoid(gate) w o / rms(o).  The
// RMS spans the 128 columns, i.e. all eight warps: the outputs of a staged
// block go to shared memory and are normalised and gated after the block,
// one barrier per block instead of one per token.
struct SpecEdges {
  const float *A_log;  // [H][128] Eq. 5 log-scales
  float g_min;
  const void *gate;    // [B][H][W][128] Eq. 6 output gate (dtype of the inputs)
  const float *rms_w;  // [H][128] RMSNorm weights
  float eps;
};

// kSplit: CTAs per chain.  The recurrence is independent across value columns
// (a column of S needs only k, g, beta and its own v), so the plain loop runs
// each chain as two CTAs of 64 columns: four smaller CTAs per SM instead of two
// overlap one CTA's state transfers with another's window better (each stages
// the window's q, k, g in full).  The fused loop keeps one CTA per chain: its
// RMS spans all 128 columns.
template <typename TIn, bool kFused, int kSplit>
__global__ void __launch_bounds__(kWarps * 32 / kSplit, 2 * kSplit)
    spec_replay_verify_d128_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                                   const TIn *__restrict__ v, const TIn *__restrict__ g,
                                   const TIn *__restrict__ beta, float *S, TIn *__restrict__ o,
                                   const int *__restrict__ n_replay, int H, int W, float scale,
                                   const SpecEdges ed) {
  static_assert(!kFused || kSplit == 1, "the fused edge needs every column of a token in one CTA");
  constexpr int kW = kWarps / kSplit;  // warps of this CTA
  const int bh = blockIdx.x / kSplit, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = lane >> 2, cg = lane & 3;
  // float4 column index of this thread (columns 4*col4 .. +3)
  const int col4 = 4 * warp + cg + (kD / 4 / kSplit) * (int)(blockIdx.x % kSplit);
  // staged window block: per token and row {alpha, k} and q; v; beta; q.k
  __shared__ float2 sak[kWB][kD];
  __shared__ float sq[kWB][kD], sv[kWB][kD], sb[kWB], sqk[kWB];
  __shared__ float so[kFused ? kWB : 1][kD];  // fused: the block's verified outputs (scaled o)

  const int nr = min(max(n_replay[bh / H], 0), W);
  float4 *S4 = reinterpret_cast<float4 *>(S + (size_t)bh * kD * kD);
  float4 s[kRowsPT];
#pragma unroll
  for (int r = 0; r < kRowsPT; ++r) s[r] = S4[(rg + 8 * r) * (kD / 4) + col4];  // in flight while staging

  for (int t0 = 0; t0 < W; t0 += kWB) {
    const int nb = min(kWB, W - t0);
    if (t0 > 0) __syncthreads();  // every warp is done with the previous block
    for (int e = tid; e < nb * kD; e += kW * 32) {
      const int u = e / kD, i = e % kD;
      const size_t in = ((size_t)bh * W + t0 + u) * kD + i;
      float gi = to_f(g[in]);
      if (kFused) gi = __fdividef(ed.g_min, 1.f + __expf(-__expf(ed.A_log[(size_t)(bh % H) * kD + i]) * gi));
      sak[u][i] = make_float2(expf(gi), to_f(k[in]));
      sq[u][i] = to_f(q[in]);
      sv[u][i] = to_f(v[in]);
    }
    if (tid < nb) sb[tid] = to_f(beta[(size_t)bh * W + t0 + tid]);
    __syncthreads();
    for (int u = warp; u < nb; u += kW) {  // q . k of token u
      float acc = 0.f;
#pragma unroll
      for (int i = lane; i < kD; i += 32) acc += sq[u][i] * sak[u][i].y;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) sqk[u] = acc;
    }
    __syncthreads();
    for (int u = 0; u < nb; ++u) {
      const int t = t0 + u;
      const bool out = t >= nr;  // bonus / draft token: its output is verified
      float2 p0 = make_float2(0.f, 0.f), p1 = p0, r0 = p0, r1 = p0;
#pragma unroll
      for (int r = 0; r < kRowsPT; ++r) {
        const float2 ak = sak[u][rg + 8 * r];
        const float2 a = make_float2(ak.x, ak.x), ka = make_float2(ak.y, ak.y);
        const float2 x0 = __fmul2_rn(a, lo2(s[r])), x1 = __fmul2_rn(a, hi2(s[r]));
        s[r] = make_float4(x0.x, x0.y, x1.x, x1.y);
        p0 = __ffma2_rn(ka, x0, p0);
        p1 = __ffma2_rn(ka, x1, p1);
        if (out) {
          const float qi = sq[u][rg + 8 * r];
          const float2 qa = make_float2(qi, qi);
          r0 = __ffma2_rn(qa, x0, r0);
          r1 = __ffma2_rn(qa, x1, r1);
        }
      }
      // column sums over the 8 row groups (lane bits 2-4): butterfly, every lane gets the total
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        p0.x += __shfl_xor_sync(0xffffffffu, p0.x, off);
        p0.y += __shfl_xor_sync(0xffffffffu, p0.y, off);
        p1.x += __shfl_xor_sync(0xffffffffu, p1.x, off);
        p1.y += __shfl_xor_sync(0xffffffffu, p1.y, off);
        if (out) {
          r0.x += __shfl_xor_sync(0xffffffffu, r0.x, off);
          r0.y += __shfl_xor_sync(0xffffffffu, r0.y, off);
          r1.x += __shfl_xor_sync(0xffffffffu, r1.x, off);
          r1.y += __shfl_xor_sync(0xffffffffu, r1.y, off);
        }
      }
      const float b = sb[u];
      const float4 vj = *reinterpret_cast<const float4 *>(&sv[u][4 * col4]);
      const float2 u0 = make_float2(b * (vj.x - p0.x), b * (vj.y - p0.y));
      const float2 u1 = make_float2(b * (vj.z - p1.x), b * (vj.w - p1.y));
      // the state after the window's last token is neither committed nor read
      // by any output (o needs only r and u), unless that token is replayed
      if (t + 1 < W || t == nr - 1) {
#pragma unroll
        for (int r = 0; r < kRowsPT; ++r) {
          const float ki1 = sak[u][rg + 8 * r].y;
          const float2 ki = make_float2(ki1, ki1);
          const float2 x0 = __ffma2_rn(ki, u0, lo2(s[r])), x1 = __ffma2_rn(ki, u1, hi2(s[r]));
          s[r] = make_float4(x0.x, x0.y, x1.x, x1.y);
        }
      }
      if (t == nr - 1)  // the last accepted token: this state is committed
#pragma unroll
        for (int r = 0; r < kRowsPT; ++r) S4[(rg + 8 * r) * (kD / 4) + col4] = s[r];
      if (out && rg == 0) {
        const float qk = sqk[u];
        const float4 ov = make_float4(scale * (r0.x + qk * u0.x), scale * (r0.y + qk * u0.y),
                                      scale * (r1.x + qk * u1.x), scale * (r1.y + qk * u1.y));
        if (kFused) {
          *reinterpret_cast<float4 *>(&so[kFused ? u : 0][4 * col4]) = ov;
        } else {
          TIn *ob = o + ((size_t)bh * W + t) * kD + 4 * col4;
          put(ob + 0, ov.x);
          put(ob + 1, ov.y);
          put(ob + 2, ov.z);
          put(ob + 3, ov.w);
        }
      }
    }
    if (kFused) {
      // Eq. 6 edge of the block's verified outputs: one warp per token, four columns per lane
      __syncthreads();
      for (int u = warp; u < nb; u += kW) {
        const int t = t0 + u;
        if (t < nr) continue;
        const float4 ov = *reinterpret_cast<const float4 *>(&so[kFused ? u : 0][4 * lane]);
        float ss = (ov.x * ov.x + ov.y * ov.y) + (ov.z * ov.z + ov.w * ov.w);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rinv = rsqrtf(ss * (1.f / kD) + ed.eps);
        const size_t at = ((size_t)bh * W + t) * kD + 4 * lane;
        const TIn *gt = reinterpret_cast<const TIn *>(ed.gate) + at;
        const float *wv = ed.rms_w + (size_t)(bh % H) * kD + 4 * lane;
        const float y[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          put(o + at + j, y[j] * rinv * wv[j] * __fdividef(1.f, 1.f + __expf(-to_f(gt[j]))));
      }
    }
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
  if (a.dk == kD && a.dv == kD) {
    const SpecEdges ed{a.A_log, a.g_min, a.gate, a.rms_w, a.eps};
    if (a.gate)
      spec_replay_verify_d128_kernel<TIn, true, 1><<<a.B * a.H, kWarps * 32, 0, st>>>(
          (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.g, (const TIn *)a.beta, a.S,
          (TIn *)a.o, a.n_replay, a.H, a.W, a.scale, ed);
    else
      spec_replay_verify_d128_kernel<TIn, false, 2><<<a.B * a.H * 2, kWarps * 32 / 2, 0, st>>>(
          (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.g, (const TIn *)a.beta, a.S,
          (TIn *)a.o, a.n_replay, a.H, a.W, a.scale, ed);
    return cudaGetLastError();
  }
  if (a.gate) return cudaErrorInvalidValue;  // the fused edges exist for dk = dv = 128 only
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
