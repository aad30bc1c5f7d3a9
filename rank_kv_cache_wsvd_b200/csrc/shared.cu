// Conventional (shared-latent) SVD decode, the comparison path of the WSVD
// summaries (Japanese §1, German §1): one fp16 latent [L][R] per sequence is
// shared by all heads, and every head projects its query through its own
// B_Kh (R x Hd) and re-reads the whole shared latent.  This file holds the
// query projection q'_h = B_Kh . q_h (R values per (b, h)); the streaming part
// is the split-L kernel of decode.cu run over R-wide fp16 rows with
// heads_share = 1, and the merge + B_Vh up-projection is combine_kernel.
#include "common.cuh"

namespace wsvd {

__global__ void __launch_bounds__(256) shared_qproj_kernel(int H, int Hd, int R, const void* q, int q_dtype,
                                                           const __half* Bk, float* qglobal) {
  const int bh = blockIdx.x, h = bh % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float qr[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    qr[k] = (lane + 32 * k < Hd) ? load_q_elem(q, q_dtype, (size_t)bh * Hd + lane + 32 * k) : 0.f;
  const __half* Bh = Bk + (size_t)h * R * Hd;
  for (int j = warp; j < R; j += 8) {
    float d = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (lane + 32 * k < Hd) d = fmaf(__half2float(Bh[(size_t)j * Hd + lane + 32 * k]), qr[k], d);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) qglobal[(size_t)bh * R + j] = d;
  }
}

cudaError_t launch_shared_qproj(int B, int H, int Hd, int R, const void* q, int q_dtype, const __half* Bk,
                                float* qglobal, cudaStream_t stream) {
  shared_qproj_kernel<<<B * H, 256, 0, stream>>>(H, Hd, R, q, q_dtype, Bk, qglobal);
  return cudaGetLastError();
}

}  // namespace wsvd
