// Weight preparation: fold an orthogonal rotation S2 of each head's latent
// space into the low-rank factors, A' = A . S2 and B' = S2^T . B (the WSVD
// summaries' "Outlier-Smoothing" transforms S1, S2, German §2.C and Arabic
// §2.c: S2 is learned jointly with A and B; here it is given).  Because
// S2 . S2^T = I, c . B is unchanged while the cache holds the rotated latents
// c . S2 that are quantised.  Runs once per model load, not per token: one
// thread per output element, an fp32 dot product over r, rounded once to fp16.
#include "common.cuh"

namespace wsvd {

namespace {

// A'[h][e][j] = sum_i A[h][e][i] * S2[h][i][j]
__global__ void fold_a_kernel(int E, int r, const __half* A, const float* S2, __half* Aout) {
  const int h = blockIdx.y;
  const size_t n = (size_t)E * r;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
    const size_t e = idx / r;
    const int j = (int)(idx % r);
    const __half* a = A + ((size_t)h * E + e) * r;
    const float* s = S2 + (size_t)h * r * r + j;
    float acc = 0.f;
    for (int i = 0; i < r; ++i) acc = fmaf(__half2float(a[i]), s[(size_t)i * r], acc);
    Aout[((size_t)h * E + e) * r + j] = __float2half_rn(acc);
  }
}

// B'[h][j][d] = sum_i S2[h][i][j] * B[h][i][d]
__global__ void fold_b_kernel(int r, int Hd, const __half* B, const float* S2, __half* Bout) {
  const int h = blockIdx.y;
  const size_t n = (size_t)r * Hd;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(idx / Hd), d = (int)(idx % Hd);
    const __half* b = B + (size_t)h * r * Hd + d;
    const float* s = S2 + (size_t)h * r * r + j;
    float acc = 0.f;
    for (int i = 0; i < r; ++i) acc = fmaf(s[(size_t)i * r], __half2float(b[(size_t)i * Hd]), acc);
    Bout[((size_t)h * r + j) * Hd + d] = __float2half_rn(acc);
  }
}

// Byte ranges [p, p + n) and [q, q + m) share at least one byte.
inline bool overlap(const void* p, size_t n, const void* q, size_t m) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  return a < b + m && b < a + n;
}

inline unsigned grid_x(size_t n) { return (unsigned)std::min<size_t>((n + 255) / 256, 1024); }

}  // namespace

}  // namespace wsvd

extern "C" int wsvd_fold_latent_rotation(int H, int E, int r, int Hd, const float* S2_k, const float* S2_v,
                                         const void* A_k, const void* A_v, const void* B_k, const void* B_v,
                                         void* A_k_out, void* A_v_out, void* B_k_out, void* B_v_out, void* stream) {
  using namespace wsvd;
  if (H < 1 || E < 1 || r < 1 || r > 128 || Hd < 1 || H > 65535) return WSVD_ERR_INVALID_ARG;
  if (!S2_k || !S2_v || !A_k || !A_v || !B_k || !B_v || !A_k_out || !A_v_out || !B_k_out || !B_v_out)
    return WSVD_ERR_INVALID_ARG;
  // No output may share a byte with any input or with another output.
  const size_t na = (size_t)H * E * r * 2, nb = (size_t)H * r * Hd * 2, ns = (size_t)H * r * r * 4;
  const void* outs[4] = {A_k_out, A_v_out, B_k_out, B_v_out};
  const size_t out_n[4] = {na, na, nb, nb};
  const void* ins[6] = {A_k, A_v, B_k, B_v, S2_k, S2_v};
  const size_t in_n[6] = {na, na, nb, nb, ns, ns};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 6; ++i)
      if (overlap(outs[o], out_n[o], ins[i], in_n[i])) return WSVD_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlap(outs[o], out_n[o], outs[o2], out_n[o2])) return WSVD_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();  // the status below is these launches', not an earlier call's
  const dim3 ga(grid_x((size_t)E * r), H), gb(grid_x((size_t)r * Hd), H);
  fold_a_kernel<<<ga, 256, 0, s>>>(E, r, static_cast<const __half*>(A_k), S2_k, static_cast<__half*>(A_k_out));
  fold_a_kernel<<<ga, 256, 0, s>>>(E, r, static_cast<const __half*>(A_v), S2_v, static_cast<__half*>(A_v_out));
  fold_b_kernel<<<gb, 256, 0, s>>>(r, Hd, static_cast<const __half*>(B_k), S2_k, static_cast<__half*>(B_k_out));
  fold_b_kernel<<<gb, 256, 0, s>>>(r, Hd, static_cast<const __half*>(B_v), S2_v, static_cast<__half*>(B_v_out));
  return cudaGetLastError() == cudaSuccess ? WSVD_OK : WSVD_ERR_CUDA;
}
