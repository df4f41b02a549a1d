// Internal launch interface between the C-ABI layer (kda_api.cu) and the
// kernels.  Not installed; the public interface is include/kda.h.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

// Device status word codes (written by kernels, read by kda_get_device_status).
enum : unsigned { kDevOk = 0, kDevTimeout = 1, kDevBounds = 2 };

// Address of the status word on the current device.
unsigned *device_status_ptr();

struct ChunkArgs {
  const void *q, *k, *v, *g, *beta;
  const float *h0;
  void *o;
  float *hT;
  int B, H, T, dk, dv;
  int bf16;     // 1: q,k,v,g,beta,o are bf16; 0: fp32
  float scale;  // resolved (> 0)
  unsigned *status;
  void *workspace;  // scratch of at least the planned size (context-parallel passes)
  int segments;     // in-device context-parallel segments per chain (1 = none)
  float *ckpt;        // [B*H][n_ckpt][dk][dv] state checkpoints, or null
  int ckpt_interval;  // tokens between checkpoints (multiple of 64) when ckpt is set
  int n_ckpt;         // T / ckpt_interval
  const float *A_log;  // [H][dk] decay log-scales when `g` holds the logits z (fused Eq. 5 gate), else null
  float g_min;         // lower bound of the fused gate
  uint64_t wait_ns;    // wall-time limit of the tensor-core kernel's bounded waits
  int stall;           // failure-detection tests: make a wait run out (kda_debug_inject_stall)
  const void *gate;    // [B][H][T][dv] output gate of the fused Eq. 6 edge (o then holds y), or null
  const float *rms_w;  // [H][dv] RMSNorm weights of that edge
  float eps;
};

// Failure-detection test settings (kda_debug_set_wait_limit, kda_debug_inject_stall).
uint64_t debug_wait_ns();
int debug_stall();

struct DecodeArgs {
  const void *q, *k, *v, *g, *beta;
  float *S;
  void *o;
  int B, H, dk, dv;
  int bf16;
  float scale;
};

struct OutGateArgs {
  const void *o, *gate;
  const float *w;  // [H][dv] RMSNorm weights
  void *y;
  int B, H, T, dv;
  int bf16;
  float eps;
};

struct SpecArgs {
  const void *q, *k, *v, *g, *beta;
  float *S;
  void *o;
  const int *n_replay;  // [B] accepted tokens to replay per sequence (device)
  int B, H, W, dk, dv;
  int bf16;
  float scale;
  // fused gate edges (kda_spec_replay_verify_fused; gate == null: plain loop):
  // g holds the Eq. 5 logits z, o receives the Eq. 6 edge y
  const float *A_log;
  float g_min;
  const void *gate;
  const float *rms_w;
  float eps;
};

cudaError_t launch_spec_replay_verify(const SpecArgs &a, cudaStream_t s);
cudaError_t launch_out_gate(const OutGateArgs &a, cudaStream_t s);
cudaError_t launch_kcp_compose(const float *M, const float *St, const float *h0, float *S_in, int R, int BH, int dk,
                               int dv, cudaStream_t s);
cudaError_t launch_chunk_simt16(const ChunkArgs &a, cudaStream_t s);
cudaError_t launch_chunk_tc32(const ChunkArgs &a, cudaStream_t s);
// Segment transition of every chain over its T tokens (kda_chunk_transition):
// St [BH][128][128] the end state from zero, M [BH][128][128] row-major.
cudaError_t launch_chunk_tc32_transition(const ChunkArgs &a, float *St, float *M, cudaStream_t s);
// Planning of the tensor-core path: segments per chain, segment length, workspace bytes.
void tc32_plan(int BH, int T, int *segments, int *seg_len);
int tc32_segments(int BH, int T);
size_t tc32_workspace(int BH, int T);
cudaError_t launch_recurrent_step(const DecodeArgs &a, cudaStream_t s);

}  // namespace kda
