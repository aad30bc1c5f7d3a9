// Internal declarations shared by the kernel translation units and the C ABI layer.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/wsvd.h"

namespace wsvd {

// Pipeline waits give up after one second of wall time (see mbar_wait_bounded).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Split-L decode: 8 consumer warps + 1 producer warp per CTA.
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kDecodeThreads = kConsumerThreads + 32;   // cluster kernel: + producer warp
constexpr int kPersistThreads = kConsumerThreads + 64;  // persistent kernel: + producer and helper warps
// Upper bound on the persistent grid; sizes the partial-result workspace.
constexpr int kMaxDecodeCtas = 2048;

enum Codec { kCodecI8 = 0, kCodecI4 = 1, kCodecF16 = 2 };
enum QMode { kQProj = 0, kQDirect = 1, kQGlobal = 2 };

// Arguments of the persistent split-L decode kernel (one struct for every codec).
struct DecodeArgs {
  int B, H, Hd, W;       // W: latent width per token (r, Hd or R)
  int L_cap;
  int ctas;              // persistent grid size C (set by launch_decode)
  int dep;               // programmatic dependency: 0 none, 1 only q' (qglobal), 2 everything (set by launch_decode)
  int heads_share;       // 1: the latent rows of (b, h) are the rows of b (shared-latent path)
  const int32_t* seq_lens;
  const void* q;
  int q_dtype;
  const uint8_t* lat_k;  // rows of W codes / values
  const uint8_t* lat_v;
  const __half* scale_k; // per-token scales (quantised codecs only)
  const __half* scale_v;
  const void* Bk;        // [H][W][Hd] fp16, or int8 when w8
  const void* Bv;        // [H][W][Hd] fp16, or int8 when w8; nullptr for the dense path (W == Hd)
  const float* sBk;      // w8: per-column scales [H][Hd] of B_k (B_k[h][j][d] * sBk[h][d])
  const float* sBv;      // w8: per-column scales [H][Hd] of B_v
  int w8;                // 1: B_k, B_v are int8 with per-column fp32 scales
  float* qglobal;        // [B][H][W] projected q' (kQGlobal; workspace)
  float qscale;          // softmax_scale * log2(e)
  float* out;            // [B][H][Hd]
  float* partials;       // [(kMaxDecodeCtas + B*H)][W + 2]
  int32_t* counters;     // [B*H], zero between calls
  int32_t* err;
};

// Host launchers (decode.cu, shared.cu, append.cu).  Return a cudaError_t.
bool decode_supported(int codec, int rowbytes, int qmode);
// after_append: the preceding kernel in `stream` writes the cache (the fused
// step); the decode is launched as its programmatic dependent and reads q and
// the B matrices before that kernel completes.  The persistent path launches
// the q' projection first (launch_qproj) and the decode behind it.
cudaError_t launch_decode(int codec, int rowbytes, int qmode, DecodeArgs a, cudaStream_t stream,
                          bool after_append = false);
// q'[b][h][:] = B_Kh . q[b, h] (W values) into qglobal.  after_append: launched
// as a programmatic dependent of the preceding kernel, and completes only
// after that kernel has (so a decode launched behind it may rely on both).
cudaError_t launch_qproj(int B, int H, int Hd, int W, const void* q, int q_dtype, const void* Bk, const float* sBk,
                         int w8, float* qglobal, cudaStream_t stream, bool after_append);
// Kernels one launch_decode call issues (1, or 2 with the q' projection).
int decode_launch_count(int codec, int rowbytes, int qmode, const DecodeArgs& a);

struct AppendArgs {
  int B, H, E, r, bits, L_cap, blk, cluster;
  float hnorm;           // 1/sqrt(blk), correctly rounded
  const void* x;
  int x_dtype;
  const void* Ak;        // [H][E][r] fp16, or int8 when w8
  const void* Av;
  const float* sAk;      // w8: per-column scales [H][r] (A_k[h][e][j] * sAk[h][j])
  const float* sAv;
  int w8;                // 1: A_k, A_v are int8 with per-column fp32 scales
  int32_t* seq_lens;
  uint8_t* lat_k;
  uint8_t* lat_v;
  __half* scale_k;
  __half* scale_v;
  int32_t* counter;
  int32_t* err;
  int dep;               // 1: launched as a programmatic dependent of the grid that writes x (read after the wait)
};
int append_cluster_size(int E, int blk);
// wsvd_decode_attention with caller-provided scratch that is NOT zero on entry
// (the no-allocation entry point's static array): validates every argument
// exactly as wsvd_decode_attention does, and only then clears the per-(b, h)
// counters (an asynchronous memset on `stream`) and launches.  Nothing is
// queued when validation fails.
int decode_with_scratch(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens, const void* q,
                        int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                        const void* scale_v, const void* B_k, const void* B_v, float softmax_scale, float* out,
                        void* scratch, size_t scratch_bytes, int32_t* err, cudaStream_t stream);
size_t append_smem_bytes(int B, int E, int r, int cluster);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);
// The append and the decode of one step as one cluster grid (decode.cu), for
// one sequence on the cluster decode path; same results as launch_append then
// launch_decode(after_append).  When the shapes do not allow it nothing is
// queued and *launched is false.
bool step_fused_applies(const AppendArgs& ap, const DecodeArgs& a);
cudaError_t launch_step_fused(const AppendArgs& ap, const DecodeArgs& a, cudaStream_t stream, bool* launched);

}  // namespace wsvd
