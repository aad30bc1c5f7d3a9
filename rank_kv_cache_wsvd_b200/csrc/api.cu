// C ABI of the library: host-side validation, split planning and launches.
// No allocation, no synchronisation; every launch goes to the caller's stream.
// (The captured host-buffer step is the one exception: creating it builds and
// instantiates a CUDA graph, once.)
#include <math.h>

#include <algorithm>
#include <new>

#include "common.cuh"
#include "wsvd_internal.h"

using namespace wsvd;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline float resolve_scale(float softmax_scale, int Hd) {
  return softmax_scale != 0.f ? softmax_scale : (float)(1.0 / sqrt((double)Hd));
}

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Decode workspace: split partials (m, l, o[W]) for every slot a persistent
// grid can use, one completion counter per (b, h), then the projected query
// q' [B][H][W] fp32 of the persistent path.
inline size_t partial_bytes(int B, int H, int W) {
  return align16(((size_t)kMaxDecodeCtas + (size_t)B * H) * ((size_t)W + 2) * sizeof(float));
}
inline size_t counter_bytes(int B, int H) { return align16((size_t)B * H * 4); }
inline size_t decode_ws_bytes(int B, int H, int W) {
  return partial_bytes(B, H, W) + counter_bytes(B, H) + align16((size_t)B * H * W * sizeof(float));
}

// Carve the caller's decode workspace into the kernel's regions.
void bind_workspace(DecodeArgs* a, void* workspace) {
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a->partials = reinterpret_cast<float*>(w);
  a->counters = reinterpret_cast<int32_t*>(w + partial_bytes(a->B, a->H, a->W));
  a->qglobal = reinterpret_cast<float*>(w + partial_bytes(a->B, a->H, a->W) + counter_bytes(a->B, a->H));
}

// Device address of pinned host memory that is mapped into the device's
// address space (every cudaHostAlloc / cudaMallocHost allocation under unified
// addressing), or nullptr for any other pointer.
void* mapped_device_pointer(const void* host) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

// The step's inputs from mapped host memory into the step workspace, 16 bytes
// per thread and load, uncached (the host rewrites these buffers every step).
// The append is launched behind it as a programmatic dependent: it streams its
// weights at once and reads x after griddepcontrol.wait.
__global__ void __launch_bounds__(256) step_ingest_kernel(const uint4* x_src, uint4* x_dst, int nx, const uint4* q_src,
                                                          uint4* q_dst, int nq) {
  griddep_launch_dependents();
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nx + nq; i += stride) {
    if (i < nx) x_dst[i] = __ldcv(x_src + i);
    else q_dst[i - nx] = __ldcv(q_src + (i - nx));
  }
}

constexpr size_t kAppendWorkspaceBytes = 256;  // the completion counter (padded)

// Shared validation of the decode entry points.
int check_common(int B, int H, int Hd, int L_cap, const int32_t* seq_lens, const void* q, int q_dtype,
                 const float* out, const void* workspace) {
  if (B < 0 || H < 1 || L_cap < 0) return WSVD_ERR_INVALID_ARG;
  if (B == 0) return WSVD_OK;
  if (B > 4096) return WSVD_ERR_UNSUPPORTED;
  if (Hd != 32 && Hd != 64 && Hd != 128 && Hd != 256) return WSVD_ERR_UNSUPPORTED;
  if (L_cap % 8) return WSVD_ERR_UNSUPPORTED;
  if (q_dtype != WSVD_DTYPE_FP16 && q_dtype != WSVD_DTYPE_BF16) return WSVD_ERR_INVALID_ARG;
  if (!seq_lens || !q || !out || !workspace) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return WSVD_ERR_INVALID_ARG;
  return WSVD_OK;
}

int run_decode(int codec, int rowbytes, int qmode, DecodeArgs a, void* workspace, cudaStream_t stream) {
  bind_workspace(&a, workspace);
  if (launch_decode(codec, rowbytes, qmode, a, stream) != cudaSuccess) return WSVD_ERR_CUDA;
  return WSVD_OK;
}


// Validation and argument set-up of wsvd_decode_attention (shared with the
// fused step).  Returns WSVD_OK with *a filled, or an error status.
int prepare_wsvd_decode(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens, const void* q,
                        int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                        const void* scale_v, const void* B_k, const void* B_v, const float* sB_k, const float* sB_v,
                        int w8, float softmax_scale, float* out, void* workspace, size_t workspace_bytes, int32_t* err,
                        DecodeArgs* a) {
  int st = check_common(B, H, Hd, L_cap, seq_lens, q, q_dtype, out, workspace);
  if (st != WSVD_OK || B == 0) return st;
  if (bits != 8 && bits != 4) return WSVD_ERR_INVALID_ARG;
  if (r < 1 || (r * bits) % 8) return WSVD_ERR_INVALID_ARG;
  const int rowbytes = r * bits / 8;
  if (!decode_supported(bits == 8 ? kCodecI8 : kCodecI4, rowbytes, kQProj)) return WSVD_ERR_UNSUPPORTED;
  if (!lat_k || !lat_v || !scale_k || !scale_v || !B_k || !B_v) return WSVD_ERR_INVALID_ARG;
  if (w8 && (!sB_k || !sB_v)) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(lat_k) || !aligned16(lat_v) || !aligned16(scale_k) || !aligned16(scale_v) ||
      !aligned16(B_k) || !aligned16(B_v))
    return WSVD_ERR_INVALID_ARG;
  if (w8 && (!aligned16(sB_k) || !aligned16(sB_v))) return WSVD_ERR_INVALID_ARG;  // staged by bulk copies
  if (workspace_bytes < decode_ws_bytes(B, H, r)) return WSVD_ERR_WORKSPACE_TOO_SMALL;
  a->B = B; a->H = H; a->Hd = Hd; a->W = r; a->L_cap = L_cap; a->heads_share = 0;
  a->seq_lens = seq_lens; a->q = q; a->q_dtype = q_dtype;
  a->lat_k = lat_k; a->lat_v = lat_v;
  a->scale_k = static_cast<const __half*>(scale_k); a->scale_v = static_cast<const __half*>(scale_v);
  a->Bk = B_k; a->Bv = B_v; a->sBk = sB_k; a->sBv = sB_v; a->w8 = w8;
  a->qscale = resolve_scale(softmax_scale, Hd) * 1.4426950408889634f;
  a->out = out; a->err = err;
  return WSVD_OK;
}

// Validation and argument set-up of wsvd_latent_append (shared with the fused step).
int prepare_append(int B, int H, int E, int r, int bits, int L_cap, int hadamard_block, const void* x, int x_dtype,
                   const void* A_k, const void* A_v, const float* sA_k, const float* sA_v, int w8,
                   int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, void* workspace,
                   size_t workspace_bytes, int32_t* err, AppendArgs* a) {
  if (B < 0 || H < 1 || E < 1 || r < 1 || L_cap < 0) return WSVD_ERR_INVALID_ARG;
  if (B == 0) return WSVD_OK;
  if (bits != 8 && bits != 4) return WSVD_ERR_INVALID_ARG;
  if (x_dtype != WSVD_DTYPE_FP16 && x_dtype != WSVD_DTYPE_BF16) return WSVD_ERR_INVALID_ARG;
  if (hadamard_block < 1 || hadamard_block > 1024 || (hadamard_block & (hadamard_block - 1)))
    return WSVD_ERR_INVALID_ARG;
  if (E % hadamard_block) return WSVD_ERR_INVALID_ARG;
  // r / 8 column groups of 8 must divide a warp (the row walk and the lane reduction)
  if (B > 16 || (r != 8 && r != 16 && r != 32 && r != 64 && r != 128) || (r * bits / 8) % 4 || E > 65536)
    return WSVD_ERR_UNSUPPORTED;
  if (!x || !A_k || !A_v || !seq_lens || !lat_k || !lat_v || !scale_k || !scale_v || !workspace)
    return WSVD_ERR_INVALID_ARG;
  if (w8 && (!sA_k || !sA_v)) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(A_k) || !aligned16(A_v) || !aligned16(lat_k) || !aligned16(lat_v) ||
      !aligned16(scale_k) || !aligned16(scale_v) || !aligned16(workspace))
    return WSVD_ERR_INVALID_ARG;
  if (workspace_bytes < kAppendWorkspaceBytes) return WSVD_ERR_WORKSPACE_TOO_SMALL;
  const int cl = append_cluster_size(E, hadamard_block);
  if (cl < 1) return WSVD_ERR_UNSUPPORTED;
  if (append_smem_bytes(B, E, r, cl) > 200 * 1024) return WSVD_ERR_UNSUPPORTED;
  a->B = B; a->H = H; a->E = E; a->r = r; a->bits = bits; a->L_cap = L_cap; a->blk = hadamard_block;
  a->cluster = cl;
  a->hnorm = (float)(1.0 / sqrt((double)hadamard_block));
  a->x = x; a->x_dtype = x_dtype;
  a->Ak = A_k; a->Av = A_v; a->sAk = sA_k; a->sAv = sA_v; a->w8 = w8;
  a->seq_lens = seq_lens; a->lat_k = lat_k; a->lat_v = lat_v;
  a->scale_k = static_cast<__half*>(scale_k); a->scale_v = static_cast<__half*>(scale_v);
  a->counter = static_cast<int32_t*>(workspace); a->err = err;
  return WSVD_OK;
}

// The append, then the decode launched behind it as a programmatic dependent
// (shared by the fp16 and int8-weight one-call steps).
int run_step(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block, const void* x, int x_dtype,
             const void* A_k, const void* A_v, const float* sA_k, const float* sA_v, int32_t* seq_lens, uint8_t* lat_k,
             uint8_t* lat_v, void* scale_k, void* scale_v, const void* q, int q_dtype, const void* B_k,
             const void* B_v, const float* sB_k, const float* sB_v, int w8, float softmax_scale, float* out,
             void* append_workspace, size_t append_workspace_bytes, void* decode_workspace,
             size_t decode_workspace_bytes, int32_t* err, void* stream) {
  AppendArgs ap{};
  int st = prepare_append(B, H, E, r, bits, L_cap, hadamard_block, x, x_dtype, A_k, A_v, sA_k, sA_v, w8, seq_lens,
                          lat_k, lat_v, scale_k, scale_v, append_workspace, append_workspace_bytes, err, &ap);
  if (st != WSVD_OK) return st;
  DecodeArgs dp{};
  st = prepare_wsvd_decode(B, H, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v, B_k, B_v,
                           sB_k, sB_v, w8, softmax_scale, out, decode_workspace, decode_workspace_bytes, err, &dp);
  if (st != WSVD_OK || B == 0) return st;
  bind_workspace(&dp, decode_workspace);
  bool fused = false;
  if (launch_step_fused(ap, dp, as_stream(stream), &fused) != cudaSuccess) return WSVD_ERR_CUDA;
  if (fused) return WSVD_OK;
  if (launch_append(ap, as_stream(stream)) != cudaSuccess) return WSVD_ERR_CUDA;
  if (launch_decode(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, dp, as_stream(stream), true) !=
      cudaSuccess)
    return WSVD_ERR_CUDA;
  return WSVD_OK;
}

}  // namespace

int wsvd::decode_with_scratch(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens, const void* q,
                        int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                        const void* scale_v, const void* B_k, const void* B_v, float softmax_scale, float* out,
                        void* scratch, size_t scratch_bytes, int32_t* err, cudaStream_t stream) {
  DecodeArgs a{};
  const int st = prepare_wsvd_decode(B, H, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v,
                                     B_k, B_v, nullptr, nullptr, 0, softmax_scale, out, scratch, scratch_bytes, err,
                                     &a);
  if (st != WSVD_OK || B == 0) return st;
  // Only the counters must start at zero: partials and q' are written before
  // they are read.
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + partial_bytes(B, H, r), 0, counter_bytes(B, H), stream) !=
      cudaSuccess)
    return WSVD_ERR_CUDA;
  return run_decode(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, a, scratch, stream);
}

extern "C" {

const char* wsvd_status_string(int status) {
  switch (status) {
    case WSVD_OK: return "ok";
    case WSVD_ERR_INVALID_ARG: return "invalid argument";
    case WSVD_ERR_UNSUPPORTED: return "unsupported shape or format";
    case WSVD_ERR_CUDA: return "CUDA runtime error";
    case WSVD_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    default: return "unknown status";
  }
}

int wsvd_abi_version(void) { return 100; }

size_t wsvd_cache_bytes(int B, int H, int L_cap, int r, int bits) {
  if (B < 0 || H < 0 || L_cap < 0 || r < 0 || (bits != 8 && bits != 4)) return 0;
  return (size_t)B * H * L_cap * ((size_t)2 * r * bits / 8 + 2 * 2);
}

size_t shared_cache_bytes(int B, int L_cap, int R) {
  if (B < 0 || L_cap < 0 || R < 0) return 0;
  return (size_t)B * L_cap * 2 * R * 2;
}

size_t dense_cache_bytes(int B, int H, int L_cap, int Hd) {
  if (B < 0 || H < 0 || L_cap < 0 || Hd < 0) return 0;
  return (size_t)B * H * L_cap * 2 * Hd * 2;
}

size_t wsvd_decode_workspace_size(int B, int H, int r) {
  if (B < 0 || H < 0 || r < 1) return 0;
  return decode_ws_bytes(B, H, r);
}

size_t dense_decode_workspace_size(int B, int H, int Hd) {
  if (B < 0 || H < 0 || Hd < 1) return 0;
  return decode_ws_bytes(B, H, Hd);
}

size_t shared_decode_workspace_size(int B, int H, int R) {
  if (B < 0 || H < 0 || R < 1) return 0;
  return decode_ws_bytes(B, H, R);
}

int wsvd_decode_attention(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                          const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                          const void* scale_k, const void* scale_v, const void* B_k, const void* B_v,
                          float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                          int32_t* err, void* stream) {
  DecodeArgs a{};
  const int st = prepare_wsvd_decode(B, H, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v,
                                     B_k, B_v, nullptr, nullptr, 0, softmax_scale, out, workspace, workspace_bytes, err,
                                     &a);
  if (st != WSVD_OK || B == 0) return st;
  return run_decode(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, a, workspace, as_stream(stream));
}

int wsvd_decode_attention_w8(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                             const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                             const void* scale_k, const void* scale_v, const int8_t* B_k, const int8_t* B_v,
                             const float* sB_k, const float* sB_v, float softmax_scale, float* out, void* workspace,
                             size_t workspace_bytes, int32_t* err, void* stream) {
  DecodeArgs a{};
  const int st = prepare_wsvd_decode(B, H, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v,
                                     B_k, B_v, sB_k, sB_v, 1, softmax_scale, out, workspace, workspace_bytes, err, &a);
  if (st != WSVD_OK || B == 0) return st;
  return run_decode(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, a, workspace, as_stream(stream));
}

int dense_decode_attention(int B, int H, int Hd, int L_cap, const int32_t* seq_lens, const void* q, int q_dtype,
                           const void* K, const void* V, float softmax_scale, float* out, void* workspace,
                           size_t workspace_bytes, int32_t* err, void* stream) {
  int st = check_common(B, H, Hd, L_cap, seq_lens, q, q_dtype, out, workspace);
  if (st != WSVD_OK || B == 0) return st;
  const int rowbytes = Hd * 2;
  if (!decode_supported(kCodecF16, rowbytes, kQDirect)) return WSVD_ERR_UNSUPPORTED;
  if (!K || !V) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V)) return WSVD_ERR_INVALID_ARG;
  if (workspace_bytes < dense_decode_workspace_size(B, H, Hd)) return WSVD_ERR_WORKSPACE_TOO_SMALL;

  DecodeArgs a{};
  a.B = B; a.H = H; a.Hd = Hd; a.W = Hd; a.L_cap = L_cap; a.heads_share = 0;
  a.seq_lens = seq_lens; a.q = q; a.q_dtype = q_dtype;
  a.lat_k = static_cast<const uint8_t*>(K); a.lat_v = static_cast<const uint8_t*>(V);
  a.Bv = nullptr;
  a.qscale = resolve_scale(softmax_scale, Hd) * 1.4426950408889634f;
  a.out = out; a.err = err;
  return run_decode(kCodecF16, rowbytes, kQDirect, a, workspace, as_stream(stream));
}

int shared_latent_svd_decode(int B, int H, int Hd, int R, int L_cap, const int32_t* seq_lens, const void* q,
                             int q_dtype, const void* lat_k, const void* lat_v, const void* B_k, const void* B_v,
                             float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                             int32_t* err, void* stream) {
  int st = check_common(B, H, Hd, L_cap, seq_lens, q, q_dtype, out, workspace);
  if (st != WSVD_OK || B == 0) return st;
  const int rowbytes = R * 2;
  if (R < 1 || !decode_supported(kCodecF16, rowbytes, kQGlobal)) return WSVD_ERR_UNSUPPORTED;
  if (!lat_k || !lat_v || !B_k || !B_v) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(lat_k) || !aligned16(lat_v) || !aligned16(B_k) || !aligned16(B_v)) return WSVD_ERR_INVALID_ARG;
  if (workspace_bytes < shared_decode_workspace_size(B, H, R)) return WSVD_ERR_WORKSPACE_TOO_SMALL;

  DecodeArgs a{};
  a.B = B; a.H = H; a.Hd = Hd; a.W = R; a.L_cap = L_cap; a.heads_share = 1;
  a.seq_lens = seq_lens; a.q = q; a.q_dtype = q_dtype;
  a.lat_k = static_cast<const uint8_t*>(lat_k); a.lat_v = static_cast<const uint8_t*>(lat_v);
  a.Bk = static_cast<const __half*>(B_k); a.Bv = static_cast<const __half*>(B_v);
  a.qscale = resolve_scale(softmax_scale, Hd) * 1.4426950408889634f;
  a.out = out; a.err = err;
  return run_decode(kCodecF16, rowbytes, kQGlobal, a, workspace, as_stream(stream));
}

int wsvd_decode_launch_count(int B, int H, int Hd, int r, int bits, int L_cap) {
  if (B < 1 || H < 1 || L_cap < 0 || (bits != 8 && bits != 4) || r < 1 || (r * bits) % 8) return 0;
  DecodeArgs a{};
  a.B = B; a.H = H; a.Hd = Hd; a.W = r; a.L_cap = L_cap;
  return decode_launch_count(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, a);
}

int wsvd_step_launch_count(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block, int w8) {
  if (B < 1 || H < 1 || E < 1 || L_cap < 0 || (bits != 8 && bits != 4) || r < 1 || (r * bits) % 8) return 0;
  if (hadamard_block < 1 || (hadamard_block & (hadamard_block - 1)) || E % hadamard_block) return 0;
  const int cl = append_cluster_size(E, hadamard_block);
  if (cl < 1) return 0;
  DecodeArgs a{};
  a.B = B; a.H = H; a.Hd = Hd; a.W = r; a.L_cap = L_cap; a.w8 = w8 ? 1 : 0;
  AppendArgs ap{};
  ap.B = B; ap.H = H; ap.E = E; ap.r = r; ap.bits = bits; ap.L_cap = L_cap; ap.blk = hadamard_block;
  ap.cluster = cl; ap.w8 = a.w8;
  if (step_fused_applies(ap, a)) return 1;
  const int n = decode_launch_count(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, a);
  return n > 0 ? 1 + n : 0;
}

size_t wsvd_append_workspace_size(void) { return kAppendWorkspaceBytes; }

int wsvd_latent_append(int B, int H, int E, int r, int bits, int L_cap, int hadamard_block, const void* x,
                       int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens, uint8_t* lat_k,
                       uint8_t* lat_v, void* scale_k, void* scale_v, void* workspace, size_t workspace_bytes,
                       int32_t* err, void* stream) {
  AppendArgs a{};
  const int st = prepare_append(B, H, E, r, bits, L_cap, hadamard_block, x, x_dtype, A_k, A_v, nullptr, nullptr, 0,
                                seq_lens, lat_k, lat_v, scale_k, scale_v, workspace, workspace_bytes, err, &a);
  if (st != WSVD_OK || B == 0) return st;
  if (launch_append(a, as_stream(stream)) != cudaSuccess) return WSVD_ERR_CUDA;
  return WSVD_OK;
}

int wsvd_latent_append_w8(int B, int H, int E, int r, int bits, int L_cap, int hadamard_block, const void* x,
                          int x_dtype, const int8_t* A_k, const int8_t* A_v, const float* sA_k, const float* sA_v,
                          int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                          void* workspace, size_t workspace_bytes, int32_t* err, void* stream) {
  AppendArgs a{};
  const int st = prepare_append(B, H, E, r, bits, L_cap, hadamard_block, x, x_dtype, A_k, A_v, sA_k, sA_v, 1,
                                seq_lens, lat_k, lat_v, scale_k, scale_v, workspace, workspace_bytes, err, &a);
  if (st != WSVD_OK || B == 0) return st;
  if (launch_append(a, as_stream(stream)) != cudaSuccess) return WSVD_ERR_CUDA;
  return WSVD_OK;
}

int wsvd_append_and_decode(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                           const void* x, int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens,
                           uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, const void* q, int q_dtype,
                           const void* B_k, const void* B_v, float softmax_scale, float* out,
                           void* append_workspace, size_t append_workspace_bytes, void* decode_workspace,
                           size_t decode_workspace_bytes, int32_t* err, void* stream) {
  return run_step(B, H, Hd, E, r, bits, L_cap, hadamard_block, x, x_dtype, A_k, A_v, nullptr, nullptr, seq_lens,
                  lat_k, lat_v, scale_k, scale_v, q, q_dtype, B_k, B_v, nullptr, nullptr, 0, softmax_scale, out,
                  append_workspace, append_workspace_bytes, decode_workspace, decode_workspace_bytes, err, stream);
}

// Step workspace of wsvd_append_and_decode_host: the append counter, the
// decode workspace, then device copies of x, q and out.
struct StepHostLayout {
  size_t app, dec, x, q, out, total;
};
inline StepHostLayout step_host_layout(int B, int H, int Hd, int E, int r) {
  StepHostLayout l;
  l.app = 0;
  l.dec = align16(kAppendWorkspaceBytes);
  l.x = l.dec + decode_ws_bytes(B, H, r);
  l.q = l.x + align16((size_t)B * E * 2);
  l.out = l.q + align16((size_t)B * H * Hd * 2);
  l.total = l.out + align16((size_t)B * H * Hd * 4);
  return l;
}

size_t wsvd_step_host_workspace_size(int B, int H, int Hd, int E, int r) {
  if (B < 0 || H < 0 || Hd < 1 || E < 1 || r < 1) return 0;
  return step_host_layout(B, H, Hd, E, r).total;
}

int wsvd_append_and_decode_host(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                                const void* x_host, int x_dtype, const void* A_k, const void* A_v,
                                int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                                const void* q_host, int q_dtype, const void* B_k, const void* B_v,
                                float softmax_scale, float* out_host, void* step_workspace,
                                size_t step_workspace_bytes, int32_t* err, void* stream) {
  if (B < 0 || H < 1 || Hd < 1 || E < 1 || r < 1 || L_cap < 0) return WSVD_ERR_INVALID_ARG;
  if (B == 0) return WSVD_OK;
  if (!x_host || !q_host || !out_host || !step_workspace) return WSVD_ERR_INVALID_ARG;
  if (!aligned16(step_workspace)) return WSVD_ERR_INVALID_ARG;
  const StepHostLayout l = step_host_layout(B, H, Hd, E, r);
  if (step_workspace_bytes < l.total) return WSVD_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* w = static_cast<uint8_t*>(step_workspace);
  void* x_dev = w + l.x;
  void* q_dev = w + l.q;
  const size_t xbytes = (size_t)B * E * 2, qbytes = (size_t)B * H * Hd * 2, obytes = (size_t)B * H * Hd * 4;
  // Pinned (mapped) host buffers are read and written in place by the
  // kernels; any other host memory goes through copies.
  void* xm = mapped_device_pointer(x_host);
  void* qm = xm ? mapped_device_pointer(q_host) : nullptr;
  void* om = qm ? mapped_device_pointer(out_host) : nullptr;
  const bool in_place = om && aligned16(xm) && aligned16(qm) && aligned16(om) && xbytes % 16 == 0 &&
                        qbytes % 16 == 0 && (xbytes + qbytes) / 16 <= 0x7fffffffu;
  float* out_dev = in_place ? static_cast<float*>(om) : reinterpret_cast<float*>(w + l.out);
  AppendArgs ap{};
  int st = prepare_append(B, H, E, r, bits, L_cap, hadamard_block, x_dev, x_dtype, A_k, A_v, nullptr, nullptr, 0,
                          seq_lens, lat_k, lat_v, scale_k, scale_v, w + l.app, kAppendWorkspaceBytes, err, &ap);
  if (st != WSVD_OK) return st;
  DecodeArgs dp{};
  st = prepare_wsvd_decode(B, H, Hd, r, bits, L_cap, seq_lens, q_dev, q_dtype, lat_k, lat_v, scale_k, scale_v, B_k,
                           B_v, nullptr, nullptr, 0, softmax_scale, out_dev, w + l.dec, l.x - l.dec, err, &dp);
  if (st != WSVD_OK) return st;
  cudaStream_t s = as_stream(stream);
  (void)cudaGetLastError();  // the status below is these launches', not an earlier call's
  if (in_place) {
    const int nx = (int)(xbytes / 16), nq = (int)(qbytes / 16);
    const int grid = std::min(148, (nx + nq + 255) / 256);
    step_ingest_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(xm), static_cast<uint4*>(x_dev), nx,
                                            static_cast<const uint4*>(qm), static_cast<uint4*>(q_dev), nq);
    if (cudaGetLastError() != cudaSuccess) return WSVD_ERR_CUDA;
    ap.dep = 1;
  } else if (cudaMemcpyAsync(x_dev, x_host, xbytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
             cudaMemcpyAsync(q_dev, q_host, qbytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    return WSVD_ERR_CUDA;
  }
  bind_workspace(&dp, w + l.dec);
  bool fused = false;
  if (launch_step_fused(ap, dp, s, &fused) != cudaSuccess) return WSVD_ERR_CUDA;
  if (!fused && (launch_append(ap, s) != cudaSuccess ||
                 launch_decode(bits == 8 ? kCodecI8 : kCodecI4, r * bits / 8, kQProj, dp, s, true) != cudaSuccess))
    return WSVD_ERR_CUDA;
  if (!in_place && cudaMemcpyAsync(out_host, out_dev, obytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return WSVD_ERR_CUDA;
  return WSVD_OK;
}

struct wsvd_step_graph {
  cudaGraphExec_t exec;
};

int wsvd_step_host_graph_create(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                                const void* x_host, int x_dtype, const void* A_k, const void* A_v,
                                int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                                const void* q_host, int q_dtype, const void* B_k, const void* B_v,
                                float softmax_scale, float* out_host, void* step_workspace,
                                size_t step_workspace_bytes, int32_t* err, wsvd_step_graph** graph) {
  if (!graph) return WSVD_ERR_INVALID_ARG;
  *graph = nullptr;
  // Only the in-place route can be captured (a copy from pageable memory cannot).
  const size_t xbytes = (size_t)(B > 0 ? B : 0) * (E > 0 ? E : 0) * 2;
  const size_t qbytes = (size_t)(B > 0 ? B : 0) * (H > 0 ? H : 0) * (Hd > 0 ? Hd : 0) * 2;
  void* xm = x_host ? mapped_device_pointer(x_host) : nullptr;
  void* qm = q_host ? mapped_device_pointer(q_host) : nullptr;
  void* om = out_host ? mapped_device_pointer(out_host) : nullptr;
  if (B > 0 && !(xm && qm && om && aligned16(xm) && aligned16(qm) && aligned16(om) && xbytes % 16 == 0 &&
                 qbytes % 16 == 0))
    return WSVD_ERR_UNSUPPORTED;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return WSVD_ERR_CUDA;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return WSVD_ERR_CUDA;
  }
  const int st = wsvd_append_and_decode_host(B, H, Hd, E, r, bits, L_cap, hadamard_block, x_host, x_dtype, A_k, A_v,
                                             seq_lens, lat_k, lat_v, scale_k, scale_v, q_host, q_dtype, B_k, B_v,
                                             softmax_scale, out_host, step_workspace, step_workspace_bytes, err, cs);
  cudaGraph_t g = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(cs, &g);
  cudaStreamDestroy(cs);
  if (st != WSVD_OK || ce != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    (void)cudaGetLastError();
    return st != WSVD_OK ? st : WSVD_ERR_CUDA;
  }
  cudaGraphExec_t ex = nullptr;
  const cudaError_t ie = cudaGraphInstantiate(&ex, g, 0);
  cudaGraphDestroy(g);
  if (ie != cudaSuccess) return WSVD_ERR_CUDA;
  *graph = new (std::nothrow) wsvd_step_graph{ex};
  if (!*graph) {
    cudaGraphExecDestroy(ex);
    return WSVD_ERR_CUDA;
  }
  return WSVD_OK;
}

int wsvd_step_host_graph_launch(wsvd_step_graph* graph, void* stream) {
  if (!graph) return WSVD_ERR_INVALID_ARG;
  return cudaGraphLaunch(graph->exec, as_stream(stream)) == cudaSuccess ? WSVD_OK : WSVD_ERR_CUDA;
}

void wsvd_step_host_graph_destroy(wsvd_step_graph* graph) {
  if (!graph) return;
  cudaGraphExecDestroy(graph->exec);
  delete graph;
}

int wsvd_append_and_decode_w8(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                              const void* x, int x_dtype, const int8_t* A_k, const int8_t* A_v, const float* sA_k,
                              const float* sA_v, int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k,
                              void* scale_v, const void* q, int q_dtype, const int8_t* B_k, const int8_t* B_v,
                              const float* sB_k, const float* sB_v, float softmax_scale, float* out,
                              void* append_workspace, size_t append_workspace_bytes, void* decode_workspace,
                              size_t decode_workspace_bytes, int32_t* err, void* stream) {
  return run_step(B, H, Hd, E, r, bits, L_cap, hadamard_block, x, x_dtype, A_k, A_v, sA_k, sA_v, seq_lens, lat_k,
                  lat_v, scale_k, scale_v, q, q_dtype, B_k, B_v, sB_k, sB_v, 1, softmax_scale, out, append_workspace,
                  append_workspace_bytes, decode_workspace, decode_workspace_bytes, err, stream);
}

}  // extern "C"
