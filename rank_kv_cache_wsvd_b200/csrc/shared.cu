// Query projection q'_{b,h} = B_Kh . q_{b,h} (W values per (b, h)) into a
// global buffer, for the split-L kernel of decode.cu in its kQGlobal mode:
// the per-head low-rank path (W = r, the reassociated score q . K^T =
// (B_Kh . q) . lat_K^T of the WSVD summaries, German §2.A) and the
// conventional shared-latent SVD decode (W = R; Japanese §1, German §1).
#include "common.cuh"

namespace wsvd {

// Block (bh, y) computes q' elements j = 8 y + warp of one (b, h), each as a
// full-warp reduction of B_Kh[j, :] . q: every block lives about one memory
// round trip, so a decode launched behind this kernel is not kept from its SMs.
__global__ void __launch_bounds__(256) qproj_kernel(int H, int Hd, int R, const void* q, int q_dtype,
                                                    const void* Bk, const float* sBk, int w8, float* qglobal) {
  // A decode launched behind this kernel may start now; it waits for q'.
  griddep_launch_dependents();
  const int bh = blockIdx.x, h = bh % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.y * 8 + warp;
  if (j < R) {
    const size_t row = ((size_t)h * R + j) * Hd;
    float d = 0.f;
    if (w8) {  // int8 B_K: the column scale is folded into q
      const int8_t* B8 = static_cast<const int8_t*>(Bk) + row;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (lane + 32 * k < Hd) {
          const int col = lane + 32 * k;
          d = fmaf((float)B8[col], load_q_elem(q, q_dtype, (size_t)bh * Hd + col) * sBk[(size_t)h * Hd + col], d);
        }
    } else {
      const __half* Bh = static_cast<const __half*>(Bk) + row;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (lane + 32 * k < Hd) {
          const int col = lane + 32 * k;
          d = fmaf(__half2float(Bh[col]), load_q_elem(q, q_dtype, (size_t)bh * Hd + col), d);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) qglobal[(size_t)bh * R + j] = d;
  }
  // Launched behind the append (programmatic dependent launch): this grid
  // must not complete before that one, so that a decode waiting on this grid
  // also sees the appended row.  A no-op for a normal launch.
  griddep_wait();
}

cudaError_t launch_qproj(int B, int H, int Hd, int W, const void* q, int q_dtype, const void* Bk, const float* sBk,
                         int w8, float* qglobal, cudaStream_t stream, bool after_append) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * H, (W + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_append ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, qproj_kernel, H, Hd, W, q, q_dtype, Bk, sBk, w8, qglobal);
}

}  // namespace wsvd
