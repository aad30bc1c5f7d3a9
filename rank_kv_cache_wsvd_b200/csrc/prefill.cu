// Prefill latent write for sm_100a: a block of T new tokens per sequence (a
// prompt, e.g. the image tokens of a vision-language prompt) is rotated by the
// block Hadamard S1, projected through A_Kh / A_Vh and quantised into cache
// rows seq_lens[b] .. seq_lens[b] + T - 1 (WSVD summaries: German §2.A for the
// per-head projection, German §2.C for S1 and the W8A8 / W8A4 quantiser; every
// row is the one a single-token append of that token would write).
//
// Unlike the one-token append (a GEMV bound by reading A), the block is a real
// GEMM: C[M x N] = X~[M x E] . W[E x N] with M = B*T token rows and
// N = 2*H*r latent columns (K heads, then V heads), W[e][n] = A_kv[h][e][j].
// Three launches:
//   1. prefill_rotate_kernel: one CTA per token row rotates it in shared
//      memory (normalised FWHT), scales it by a power of two p_m (exact) so
//      that its largest element lies in [2^14, 2^15), and splits every value v
//      into two fp16 halves hi + lo = v to within 2^-22 relative;
//   2. prefill_gemm_kernel: 64 x 128 output tiles on the tensor cores
//      (mma.sync m16n8k16, fp16 x fp16 -> fp32), the hi and the lo operand
//      each multiplied by the same fp16 weight fragment, so that the product
//      carries the rotated activation to fp32-like precision (one fp16
//      product alone would move the codes by up to a few hundredths of a
//      step, far more than the quantiser's rounding ties allow); each 64-wide
//      k-tile of the hi half is accumulated from zero on the tensor cores and
//      added to an fp32 register total; tiles stream
//      through a three-stage cp.async ring; the epilogue stages the fp32
//      tile in shared memory, undoes p_m (exact) and quantises each
//      (token, head) row of r values with one warp: amax, fp16 scale,
//      round-half-even codes, row write;
//   3. prefill_advance_kernel: seq_lens[b] += T, or the block is refused.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc05.cuh"

namespace wsvd {

namespace {

constexpr int kRotThreads = 256;
constexpr int kBM = 64, kBN = 128, kBK = 64;
constexpr int kWarpsM = 4, kWarpsN = 4;         // 16 warps of 16 x 32 outputs
constexpr int kGemmThreads = 32 * kWarpsM * kWarpsN;
constexpr int kWM = kBM / kWarpsM;              // rows per warp
constexpr int kMI = kWM / 16;                   // m16 MMA tiles per warp
constexpr int kWN = kBN / kWarpsN;              // columns per warp
constexpr int kNI = kWN / 8;                    // n8 MMA tiles per warp
constexpr int kNJ = kWN / 16;                   // ldmatrix.x4.trans per k16 step (two n8 tiles each)
constexpr int kAPieces = kBM * kBK / 8 / kGemmThreads;   // 16-byte activation pieces per thread (hi and lo each)
constexpr int kWPieces = kBK * kBN / 8 / kGemmThreads;   // 16-byte weight pieces per thread
constexpr int kStages = 3;
constexpr int kAStride = kBK + 8;  // halves per shared row of an activation tile (144 B: the 8 rows of an
                                   // ldmatrix phase land on distinct 16-byte bank groups)
constexpr int kBStride = kBN + 8;  // halves per shared row of the weight tile (272 B, same reason)
constexpr int kCStride = kBN + 4;  // floats per shared row of the epilogue tile
constexpr int kATileHalves = kBM * kAStride;
constexpr int kBTileHalves = kBK * kBStride;
constexpr int kStageHalves = 2 * kATileHalves + kBTileHalves;  // hi, lo, weights
constexpr size_t kGemmSmem = std::max<size_t>((size_t)kStages * kStageHalves * 2, (size_t)kBM * kCStride * 4);

struct PrefillArgs {
  int B, T, M, H, E, r, bits, L_cap, N;
  const __half* xhi;  // [M][E]
  const __half* xlo;  // [M][E]
  const float* inv_p; // [M]: 1 / p_m
  const __half* Ak;   // [H][E][r]
  const __half* Av;
  const int32_t* seq_lens;
  uint8_t* lat_k;
  uint8_t* lat_v;
  __half* scale_k;
  __half* scale_v;
};

__device__ __forceinline__ float x_value(uint16_t bits16, int dtype) {
  return dtype == WSVD_DTYPE_BF16 ? __uint_as_float((uint32_t)bits16 << 16) : __half2float(__ushort_as_half(bits16));
}

// ------------------------------------------------------------------ 1. rotate + split
__global__ void __launch_bounds__(kRotThreads) prefill_rotate_kernel(const void* x, int x_dtype, int E, int blk,
                                                                     float hnorm, __half* xhi, __half* xlo,
                                                                     float* inv_p) {
  extern __shared__ __align__(16) float xs[];
  __shared__ float wmax[kRotThreads / 32];
  griddep_launch_dependents();  // the GEMM behind may set up (it waits for this grid before reading)
  const int m = blockIdx.x, tid = threadIdx.x;
  const int E4 = E / 4;  // E is a multiple of 64: rows are whole 8-byte groups of four values
  const uint2* xr = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + (size_t)m * E);
  float4* xs4 = reinterpret_cast<float4*>(xs);
  for (int i = tid; i < E4; i += kRotThreads) {
    const uint2 v = xr[i];
    xs4[i] = make_float4(x_value((uint16_t)(v.x & 0xffffu), x_dtype), x_value((uint16_t)(v.x >> 16), x_dtype),
                         x_value((uint16_t)(v.y & 0xffffu), x_dtype), x_value((uint16_t)(v.y >> 16), x_dtype));
  }
  __syncthreads();
  // Butterfly stages of distance hh = 1, 2, ..., blk/2: pairs (i, i + hh) with
  // bit hh of i clear never leave an aligned block of blk values (Sylvester
  // order).  Pair q of a stage: q's bits above log2(hh) move up by one.
  for (int sh = 0; (1 << sh) < blk; ++sh) {
    const int hh = 1 << sh;
    for (int q = tid; q < E / 2; q += kRotThreads) {
      const int i = ((q >> sh) << (sh + 1)) | (q & (hh - 1));
      const float u = xs[i], v = xs[i + hh];
      xs[i] = u + v;
      xs[i + hh] = u - v;
    }
    __syncthreads();
  }
  float amax = 0.f;
  for (int i = tid; i < E4; i += kRotThreads) {
    float4 v = xs4[i];
    v.x *= hnorm; v.y *= hnorm; v.z *= hnorm; v.w *= hnorm;
    xs4[i] = v;
    amax = fmaxf(fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y))), fmaxf(fabsf(v.z), fabsf(v.w)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = amax;
  __syncthreads();
  amax = 0.f;
#pragma unroll
  for (int w = 0; w < kRotThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
  // p = 2^k with amax * p in [2^14, 2^15) for a normal amax (amax in [2^e, 2^(e+1)));
  // k is clamped so that both 2^k and 2^-k are normal floats.
  int k = 0;
  if (amax > 0.f) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 127;
    k = max(-126, min(126, 14 - e));
  }
  const float p = __uint_as_float((uint32_t)(127 + k) << 23);
  uint2* hi4 = reinterpret_cast<uint2*>(xhi + (size_t)m * E);
  uint2* lo4 = reinterpret_cast<uint2*>(xlo + (size_t)m * E);
  auto split = [&](float v, __half& hi) {  // hi = fp16(v), returns fp16(v - hi)
    hi = __float2half_rn(v);
    return __float2half_rn(v - __half2float(hi));
  };
  for (int i = tid; i < E4; i += kRotThreads) {
    const float4 v = xs4[i];
    __half h0, h1, h2, h3;
    const __half l0 = split(v.x * p, h0), l1 = split(v.y * p, h1), l2 = split(v.z * p, h2), l3 = split(v.w * p, h3);
    hi4[i] = make_uint2((uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16),
                        (uint32_t)__half_as_ushort(h2) | ((uint32_t)__half_as_ushort(h3) << 16));
    lo4[i] = make_uint2((uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16),
                        (uint32_t)__half_as_ushort(l2) | ((uint32_t)__half_as_ushort(l3) << 16));
  }
  if (tid == 0) inv_p[m] = __uint_as_float((uint32_t)(127 - k) << 23);
}

// Register / shuffle version of the same rotation for rows of E = NT * EPT
// values (EPT a power of two in [4, 64]) and blocks of at most 32 * EPT: NT
// threads, thread i holds the EPT consecutive values i*EPT ..; butterfly
// distances below EPT stay in registers, distances EPT .. 16*EPT are lane
// exchanges inside the warp, so the only block-wide step is the maximum.
// The arithmetic per value is the shared-memory kernel's (the same adds and
// subtracts in the same stage order, the same normalisation, p_m and split),
// whatever NT.  More threads per row (fewer values each) keep more loads in
// flight per SM: the kernel is bound by the latency of its row loads.
template <int EPT, int NT>
__global__ void __launch_bounds__(NT) prefill_rotate_reg_kernel(const void* x, int x_dtype, int E, int blk,
                                                                float hnorm, __half* xhi, __half* xlo,
                                                                float* inv_p) {
  __shared__ float wmax[NT / 32];
  griddep_launch_dependents();  // the GEMM behind may set up (it waits for this grid before reading)
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const uint16_t* xr = static_cast<const uint16_t*>(x) + (size_t)m * E + (size_t)tid * EPT;
  float v[EPT];
#pragma unroll
  for (int k = 0; k < EPT; k += 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(xr + k);
    v[k] = x_value((uint16_t)(w.x & 0xffffu), x_dtype);
    v[k + 1] = x_value((uint16_t)(w.x >> 16), x_dtype);
    v[k + 2] = x_value((uint16_t)(w.y & 0xffffu), x_dtype);
    v[k + 3] = x_value((uint16_t)(w.y >> 16), x_dtype);
  }
  // distances inside the thread's EPT values
#pragma unroll
  for (int hh = 1; hh < EPT; hh <<= 1) {
    if (hh >= blk) break;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      if (i & hh) continue;
      const float u = v[i], w = v[i + hh];
      v[i] = u + w;
      v[i + hh] = u - w;
    }
  }
  // distances EPT, 2 EPT, ...: partner lane tid ^ d holds element i +- d*EPT
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    if (d * EPT >= blk) break;
    const bool upper = lane & d;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], d);
      v[i] = upper ? o - v[i] : v[i] + o;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    v[i] *= hnorm;
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) wmax[tid >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) amax = fmaxf(amax, wmax[w]);
  int k = 0;
  if (amax > 0.f) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 127;
    k = max(-126, min(126, 14 - e));
  }
  const float p = __uint_as_float((uint32_t)(127 + k) << 23);
  uint2* hi4 = reinterpret_cast<uint2*>(xhi + (size_t)m * E + (size_t)tid * EPT);
  uint2* lo4 = reinterpret_cast<uint2*>(xlo + (size_t)m * E + (size_t)tid * EPT);
#pragma unroll
  for (int i = 0; i < EPT; i += 4) {
    uint32_t hw[2], lw[2];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float t = v[i + q] * p;
      const __half h = __float2half_rn(t);
      const __half l = __float2half_rn(t - __half2float(h));
      const int wi = q >> 1, sh = 16 * (q & 1);
      if ((q & 1) == 0) {
        hw[wi] = (uint32_t)__half_as_ushort(h);
        lw[wi] = (uint32_t)__half_as_ushort(l);
      } else {
        hw[wi] |= (uint32_t)__half_as_ushort(h) << sh;
        lw[wi] |= (uint32_t)__half_as_ushort(l) << sh;
      }
    }
    hi4[i / 4] = make_uint2(hw[0], hw[1]);
    lo4[i / 4] = make_uint2(lw[0], lw[1]);
  }
  if (tid == 0) inv_p[m] = __uint_as_float((uint32_t)(127 - k) << 23);
}

// ------------------------------------------------------------------ 2. GEMM + quantise
// 16-byte cp.async; a false `valid` copies nothing and zero-fills the destination.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += a . b for one 16 x 8 x 16 tile (fp16 operands, fp32 accumulators).
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A thread's share of every k-tile's copies, fixed for the whole K loop: one
// 16-byte piece of the hi and of the lo activation tile, and two pieces of
// the weight tile (a piece is 8 consecutive latent columns of one head).  The
// sources are resolved once, so a k-tile only adds its offset.
struct CopyPlan {
  const __half* xhi[kAPieces];  // row m0 + arow of the split activations, column ach * 8
  const __half* xlo[kAPieces];
  const __half* w[kWPieces];    // weight row krow of the piece's head, its first column
  uint32_t a_dst[kAPieces], w_dst[kWPieces];
  bool a_ok[kAPieces], w_ok[kWPieces];
};

__device__ __forceinline__ CopyPlan plan_copies(const PrefillArgs& a, int m0, int n0, int tid) {
  static_assert(kAPieces * kGemmThreads * 8 == kBM * kBK && kWPieces * kGemmThreads * 8 == kBK * kBN,
                "whole pieces per thread");
  CopyPlan p;
#pragma unroll
  for (int i = 0; i < kAPieces; ++i) {
    const int idx = tid + i * kGemmThreads;
    const int arow = idx / (kBK / 8), ach = idx % (kBK / 8);
    p.a_ok[i] = m0 + arow < a.M;
    const size_t aoff = p.a_ok[i] ? (size_t)(m0 + arow) * a.E + ach * 8 : 0;
    p.xhi[i] = a.xhi + aoff;
    p.xlo[i] = a.xlo + aoff;
    p.a_dst[i] = (uint32_t)(arow * kAStride + ach * 8);
  }
  const int HR = a.H * a.r;
#pragma unroll
  for (int i = 0; i < kWPieces; ++i) {
    const int idx = tid + i * kGemmThreads;
    const int krow = idx / (kBN / 8), ch = idx % (kBN / 8);
    const int n = n0 + ch * 8;
    p.w_ok[i] = n < a.N;
    p.w[i] = a.Ak;
    if (p.w_ok[i]) {
      const int kv = n / HR, rem = n - kv * HR;
      const int h = rem / a.r, j = rem - h * a.r;
      p.w[i] = (kv ? a.Av : a.Ak) + ((size_t)h * a.E + krow) * a.r + j;
    }
    p.w_dst[i] = (uint32_t)(2 * kATileHalves + krow * kBStride + ch * 8);
  }
  return p;
}

// Stage k-tile kt.  Pieces outside the problem are zero-filled (their source
// pointers stay inside the arrays but are not read).
__device__ __forceinline__ void load_stage(const PrefillArgs& a, const CopyPlan& p, __half* st, int kt) {
  const int k0 = kt * kBK;
#pragma unroll
  for (int i = 0; i < kAPieces; ++i) {
    cp_async16_zfill(st + p.a_dst[i], p.xhi[i] + k0, p.a_ok[i]);
    cp_async16_zfill(st + kATileHalves + p.a_dst[i], p.xlo[i] + k0, p.a_ok[i]);
  }
#pragma unroll
  for (int i = 0; i < kWPieces; ++i) cp_async16_zfill(st + p.w_dst[i], p.w[i] + (size_t)k0 * a.r, p.w_ok[i]);
}

__global__ void __launch_bounds__(kGemmThreads, 1) prefill_gemm_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __half* sm = reinterpret_cast<__half*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / kWarpsN, wn = warp % kWarpsN;  // warp tile: rows wm*kWM.., columns wn*kWN..
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
  const int KT = a.E / kBK;
  const CopyPlan plan = plan_copies(a, m0, n0, tid);

  // acc: the hi half's products, k-tile by k-tile (below); acc_lo: the lo
  // half's, kept on the tensor cores over all of E (its sum is ~2^-11 of c,
  // so its drift is far below the hi half's rounding).  Separate accumulators
  // also make the hi and lo MMAs independent of each other.
  float acc[kMI][kNI][4], acc_lo[kMI][kNI][4];
#pragma unroll
  for (int i = 0; i < kMI; ++i)
#pragma unroll
    for (int j = 0; j < kNI; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[i][j][k] = acc_lo[i][j][k] = 0.f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < KT) load_stage(a, plan, sm + s * kStageHalves, s);
    cp_async_commit_group();
  }
  for (int kt = 0; kt < KT; ++kt) {
    cp_async_wait_group<kStages - 2>();  // k-tile kt has landed (this thread's copies)
    __syncthreads();                     // everyone's copies; and slot (kt - 1) % kStages is free
    {
      const int nk = kt + kStages - 1;
      if (nk < KT) load_stage(a, plan, sm + (nk % kStages) * kStageHalves, nk);
      cp_async_commit_group();
    }
    const __half* st = sm + (kt % kStages) * kStageHalves;
    const uint32_t ahi_base = smem_u32(st), alo_base = smem_u32(st + kATileHalves),
                   b_base = smem_u32(st + 2 * kATileHalves);
    // The tensor cores' fp32 accumulation is not round-to-nearest; a running
    // sum held in the MMA accumulator over all of E drifts by a fraction of an
    // ulp per MMA.  Each k-tile of the hi half therefore starts from zero
    // (four MMAs deep) and is added to the fp32 total with a rounded add.
    float part[kMI][kNI][4];
#pragma unroll
    for (int i = 0; i < kMI; ++i)
#pragma unroll
      for (int j = 0; j < kNI; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) part[i][j][k] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kBK; kk += 16) {
      uint32_t ahi[kMI][4], alo[kMI][4], bq[kNJ][4];
#pragma unroll
      for (int mi = 0; mi < kMI; ++mi) {
        const uint32_t off = (uint32_t)(((wm * kWM + mi * 16 + (lane & 15)) * kAStride + kk + (lane >> 4) * 8) * 2);
        ldmatrix_x4(ahi[mi], ahi_base + off);
        ldmatrix_x4(alo[mi], alo_base + off);
      }
#pragma unroll
      for (int nj = 0; nj < kNJ; ++nj) {
        const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = wn * kWN + nj * 16 + (lane >> 4) * 8;
        ldmatrix_x4_trans(bq[nj], b_base + (uint32_t)((krow * kBStride + col) * 2));
      }
#pragma unroll
      for (int mi = 0; mi < kMI; ++mi)
#pragma unroll
        for (int ni = 0; ni < kNI; ++ni) {
          const uint32_t b0 = bq[ni >> 1][(ni & 1) * 2], b1 = bq[ni >> 1][(ni & 1) * 2 + 1];
          mma_16816(part[mi][ni], ahi[mi], b0, b1);
          mma_16816(acc_lo[mi][ni], alo[mi], b0, b1);
        }
    }
#pragma unroll
    for (int i = 0; i < kMI; ++i)
#pragma unroll
      for (int j = 0; j < kNI; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][j][k] = __fadd_rn(acc[i][j][k], part[i][j][k]);
  }
  cp_async_wait_group<0>();
  __syncthreads();  // every warp is done with the ring: it becomes the epilogue tile
#pragma unroll
  for (int i = 0; i < kMI; ++i)
#pragma unroll
    for (int j = 0; j < kNI; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[i][j][k] = __fadd_rn(acc[i][j][k], acc_lo[i][j][k]);

  float* cs = reinterpret_cast<float*>(smem_raw);
  {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mi = 0; mi < kMI; ++mi)
#pragma unroll
      for (int ni = 0; ni < kNI; ++ni) {
        const int row = wm * kWM + mi * 16 + g, col = wn * kWN + ni * 8 + 2 * t;
        *reinterpret_cast<float2*>(cs + row * kCStride + col) = make_float2(acc[mi][ni][0], acc[mi][ni][1]);
        *reinterpret_cast<float2*>(cs + (row + 8) * kCStride + col) = make_float2(acc[mi][ni][2], acc[mi][ni][3]);
      }
  }
  __syncthreads();

  // One warp per (token row, head) unit of r columns; lane owns j = lane + 32q.
  const int Q = a.bits == 8 ? 127 : 7;
  const int RB = a.r * a.bits / 8;
  const int HR = a.H * a.r;
  const int heads = kBN / a.r;
  for (int u = warp; u < kBM * heads; u += kGemmThreads / 32) {
    const int i = u / heads, hh = u - i * heads;
    const int m = m0 + i, n = n0 + hh * a.r;
    if (m >= a.M || n >= a.N) continue;  // warp-uniform
    const int b = m / a.T, t = m - b * a.T;
    const int pos = a.seq_lens[b];
    if (pos < 0 || (long long)pos + a.T > a.L_cap) continue;  // refused block (flagged by the advance kernel)
    const int kv = n / HR, h = (n - kv * HR) / a.r;
    const float ip = a.inv_p[m];
    float cv[4];
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = lane + 32 * q;
      cv[q] = j < a.r ? cs[i * kCStride + hh * a.r + j] * ip : 0.f;
      amax = fmaxf(amax, fabsf(cv[q]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half sh = __float2half_rn(__fdiv_rn(amax, (float)Q));
    const float sc = __half2float(sh);
    const size_t row = ((size_t)b * a.H + h) * a.L_cap + pos + t;
    uint8_t* dst = (kv ? a.lat_v : a.lat_k) + row * RB;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = lane + 32 * q;
      const int code = sc > 0.f ? max(-Q, min(Q, __float2int_rn(__fdiv_rn(cv[q], sc)))) : 0;
      if (a.bits == 8) {
        if (j < a.r) dst[j] = (uint8_t)code;
      } else {
        const int hi = __shfl_down_sync(0xffffffffu, code, 1);  // column j + 1 (r is a multiple of 8)
        if (j < a.r && (lane & 1) == 0) dst[j / 2] = (uint8_t)((code & 0xF) | ((hi & 0xF) << 4));
      }
    }
    if (lane == 0) (kv ? a.scale_v : a.scale_k)[row] = sh;
  }
}

// ------------------------------------------------------------------ 2'. GEMM + quantise on tcgen05
// The same product and epilogue on the fifth-generation tensor cores, for
// shapes whose 64- or 128-column output tiles hold whole heads of one side
// (K or V): 128 x BN output tiles, one CTA each (BN = 128 when H * r allows
// and the tiles fill the device, else 64).
//   warp 4   TMA producer: per 64-wide k-tile, the hi and lo activation tiles
//            [128 x 64] (2-D tensor maps, 128-byte swizzle, K-major) and the
//            weight tile [64 x BN] as BN / NG boxes of one head's NG columns
//            (3-D tensor map over A [H][E][r], swizzle of NG * 2 bytes; the
//            operand is N-major) into a four-stage mbarrier ring;
//   warp 5   allocates tensor memory and issues (converged, one elected
//            lane) per k-tile four MMAs of the hi half into a fresh
//            accumulator (one of NH, so that it runs up to NH k-tiles ahead
//            of the epilogue) and four of the lo half into one accumulator
//            kept over all of E;
//   warps 0-3  thread t <-> output row t <-> tensor-memory lane t: add each
//            k-tile's hi sum to an fp32 register total with a round-to-nearest
//            add, then add the lo sum, undo p_m and quantise every head of the
//            row in registers (no cross-thread reduction: a thread holds whole
//            heads), writing codes and scales straight to the cache.
// Numerics are those of the mma.sync kernel above: each k-tile of the hi half
// is summed from zero on the tensor cores, k-tiles are added with rounding to
// nearest, the lo half keeps one tensor-core sum.
constexpr int kTcBM = 128, kTcBK = 64, kTcStages = 4, kTcThreads = 192;

template <int R, int BN_>
struct TcCfg {
  static constexpr int BN = BN_;                          // output columns per tile (whole heads)
  static constexpr int NG = R <= 64 ? R : 64;            // columns per weight box (one head, or half of r = 128)
  static constexpr int SW = NG == 16 ? 6 : (NG == 32 ? 4 : 2);  // descriptor swizzle: 32 / 64 / 128 bytes
  static constexpr int A_BYTES = kTcBM * kTcBK * 2;
  static constexpr int W_BYTES = kTcBK * BN * 2;
  static constexpr int STAGE = 2 * A_BYTES + W_BYTES;
  // NH fresh accumulators for the hi k-tile sums (the MMA warp runs up to NH
  // k-tiles ahead of the epilogue), then the lo accumulator: all 512 columns.
  static constexpr int NH = BN == 64 ? 6 : 3;
  static_assert(BN == 64 || BN == 128, "tile width");
  static_assert(R <= BN, "whole heads per tile");
  static constexpr int TCOLS = 512;
  static constexpr int SMEM = kTcStages * STAGE + 1024 + 256;
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle-atom alignment");
};

struct TcArgs {
  int M, T, H, bits, L_cap, KT;
  const float* inv_p;
  const int32_t* seq_lens;
  uint8_t* lat_k;
  uint8_t* lat_v;
  __half* scale_k;
  __half* scale_v;
  int32_t* err;
};

// TMA tile loads, warp-level: a converged warp calls them, one elected lane issues.
__device__ __forceinline__ void tma_load_2d_warp(uint32_t dst, const CUtensorMap* tm, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      "\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_warp(uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                                 uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
template <int R, int BN_>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_xhi, const __grid_constant__ CUtensorMap tm_xlo,
                      const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                      const TcArgs a) {
  using C = TcCfg<R, BN_>;
  constexpr int BN = C::BN, NG = C::NG, S = kTcStages;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::STAGE);
  uint64_t* empty = full + S;
  constexpr int NH = C::NH;
  uint64_t* hfull = empty + S;   // [NH] a k-tile's hi sum is in tensor memory
  uint64_t* hfree = hfull + NH;  // [NH] the epilogue has read it (128 arrivals)
  uint64_t* done = hfree + NH;   // every MMA of the tile has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  griddep_launch_dependents();  // the length advance behind may launch (it waits for this grid)
  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = blockIdx.x * kTcBM, n0 = blockIdx.y * BN;
  const int HR = a.H * R;
  const int kv = n0 >= HR ? 1 : 0, nl = n0 - kv * HR;  // tile columns within the K or the V side
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NH; ++i) {
      mbar_init(&hfull[i], 1);
      mbar_init(&hfree[i], 128);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 5) tc05::alloc(tmem_slot, C::TCOLS);
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  bool timed_out = false;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (!mbar_wait_bounded(bar, parity, timed_out ? 0ull : kWaitLimitNs)) {
      if (!timed_out) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      timed_out = true;
    }
  };
  const int KT = a.KT;

  // The producer and MMA warps run their loops converged (every lane waits,
  // one elected lane issues), so that the copies and MMAs issue at full rate.
  if (warp == 4) {  // ------------------------------------------------------ TMA producer
    const CUtensorMap* wmap = kv ? &tm_wv : &tm_wk;
    griddep_wait();  // the split activations come from the rotation grid launched before this one
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % S;
      if (kt >= S) wait(&empty[s], (uint32_t)(((kt / S) - 1) & 1));
      __syncwarp();
      const uint32_t st = base + (uint32_t)(s * C::STAGE);
      mbar_arrive_expect_tx_warp(&full[s], C::STAGE);
      tma_load_2d_warp(st, &tm_xhi, kt * kTcBK, m0, &full[s]);
      tma_load_2d_warp(st + C::A_BYTES, &tm_xlo, kt * kTcBK, m0, &full[s]);
#pragma unroll
      for (int g = 0; g < BN / NG; ++g) {
        const int col = nl + g * NG;
        tma_load_3d_warp(st + 2 * C::A_BYTES + g * (kTcBK * NG * 2), wmap, col % R, kt * kTcBK, col / R, &full[s]);
      }
    }
    for (int kt = std::max(0, KT - S); kt < KT; ++kt) wait(&full[kt % S], (uint32_t)((kt / S) & 1));
    __syncwarp();
  } else if (warp == 5) {  // ----------------------------------------------- MMA issuer
    constexpr uint32_t idesc = tc05::instr_desc(1, 0, 0, 0, 1, kTcBM, BN);
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % S;
      wait(&full[s], (uint32_t)((kt / S) & 1));
      const int hb = kt % NH;
      if (kt >= NH) wait(&hfree[hb], (uint32_t)(((kt / NH) - 1) & 1));
      __syncwarp();
      tc05::fence_after_sync();
      const uint32_t st = base + (uint32_t)(s * C::STAGE);
      const uint32_t dh = tmem + (uint32_t)(hb * BN), dl = tmem + (uint32_t)(NH * BN);
#pragma unroll
      for (int kk = 0; kk < kTcBK / 16; ++kk) {
        const uint64_t bd = tc05::smem_desc_sw(st + 2 * C::A_BYTES + kk * 32 * NG, 128 * NG, 16 * NG, C::SW);
        tc05::mma_f16_warp(dh, tc05::smem_desc_sw(st + kk * 32, 16, 1024, 2), bd, idesc, kk > 0);
        tc05::mma_f16_warp(dl, tc05::smem_desc_sw(st + C::A_BYTES + kk * 32, 16, 1024, 2), bd, idesc,
                           kt > 0 || kk > 0);
      }
      tc05::commit_warp(&empty[s]);
      tc05::commit_warp(&hfull[hb]);
    }
    tc05::commit_warp(done);
    wait(done, 0);  // every MMA has completed before the allocation is released
    __syncwarp();
  } else {  // -------------------------------------------------------- epilogue, thread = output row
    griddep_wait();  // 1 / p_m comes from the rotation grid
    const int row = tid;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float tot[BN];
#pragma unroll
    for (int c = 0; c < BN; ++c) tot[c] = 0.f;
    for (int kt = 0; kt < KT; ++kt) {
      const int hb = kt % NH;
      wait(&hfull[hb], (uint32_t)((kt / NH) & 1));
      tc05::fence_after_sync();
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 64) {  // two loads in flight per wait
        uint32_t va[32], vb[32];
        tc05::ld32(lane_base + (uint32_t)(hb * BN + c0), va);
        tc05::ld32(lane_base + (uint32_t)(hb * BN + c0 + 32), vb);
        tc05::wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          tot[c0 + c] = __fadd_rn(tot[c0 + c], __uint_as_float(va[c]));
          tot[c0 + 32 + c] = __fadd_rn(tot[c0 + 32 + c], __uint_as_float(vb[c]));
        }
      }
      tc05::fence_before_sync();
      mbar_arrive(&hfree[hb]);
    }
    wait(done, 0);
    tc05::fence_after_sync();
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t v[32];
      tc05::ld32(lane_base + (uint32_t)(NH * BN + c0), v);
      tc05::wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) tot[c0 + c] = __fadd_rn(tot[c0 + c], __uint_as_float(v[c]));
    }
    tc05::fence_before_sync();
    const int m = m0 + row;
    if (m < a.M) {
      const int b = m / a.T, t = m - b * a.T;
      const int pos = a.seq_lens[b];
      if (pos >= 0 && (long long)pos + a.T <= a.L_cap) {  // else refused (flagged by the advance kernel)
        const float ip = a.inv_p[m];
        const int Q = a.bits == 8 ? 127 : 7;
        constexpr int HEADS = BN / R < 1 ? 1 : BN / R;
#pragma unroll
        for (int hb = 0; hb < HEADS; ++hb) {
          const int h = (nl + hb * R) / R;
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < R; ++j) {
            tot[hb * R + j] *= ip;
            amax = fmaxf(amax, fabsf(tot[hb * R + j]));
          }
          const __half sh = __float2half_rn(__fdiv_rn(amax, (float)Q));
          const float sc = __half2float(sh);
          const size_t crow = ((size_t)b * a.H + h) * a.L_cap + pos + t;
          if (a.bits == 8) {
            uint32_t* dst = reinterpret_cast<uint32_t*>((kv ? a.lat_v : a.lat_k) + crow * R);
#pragma unroll
            for (int j4 = 0; j4 < R / 4; ++j4) {
              uint32_t w = 0;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int code = sc > 0.f ? max(-Q, min(Q, __float2int_rn(__fdiv_rn(tot[hb * R + 4 * j4 + k], sc)))) : 0;
                w |= ((uint32_t)code & 0xFFu) << (8 * k);
              }
              dst[j4] = w;
            }
          } else {
            uint32_t* dst = reinterpret_cast<uint32_t*>((kv ? a.lat_v : a.lat_k) + crow * (R / 2));
#pragma unroll
            for (int j8 = 0; j8 < R / 8; ++j8) {
              uint32_t w = 0;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int code = sc > 0.f ? max(-Q, min(Q, __float2int_rn(__fdiv_rn(tot[hb * R + 8 * j8 + k], sc)))) : 0;
                w |= ((uint32_t)code & 0xFu) << (4 * k);
              }
              dst[j8] = w;
            }
          }
          (kv ? a.scale_v : a.scale_k)[crow] = sh;
        }
      }
    }
  }
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, C::TCOLS);
  }
}

// Tensor maps are encoded on the host through the driver's entry point (no
// link-time dependence on the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_for(int inner_bytes) {
  return inner_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                           : (inner_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Activations [M][E] fp16: boxes of 64 columns x 128 rows, 128-byte swizzle.
bool encode_act_map(CUtensorMap* tm, const void* base, int M, int E) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)E, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)E * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)kTcBM};
  const cuuint32_t es[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weights [H][E][r] fp16 as a 3-D tensor (j, e, h): boxes of NG columns x 64 rows of one head.
bool encode_weight_map(CUtensorMap* tm, const void* base, int H, int E, int r, int NG) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)r, (cuuint64_t)E, (cuuint64_t)H};
  const cuuint64_t strides[2] = {(cuuint64_t)r * 2, (cuuint64_t)E * r * 2};
  const cuuint32_t box[3] = {(cuuint32_t)NG, (cuuint32_t)kTcBK, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(NG * 2), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, int BN>
cudaError_t launch_tc(const PrefillArgs& pa, const void* A_k, const void* A_v, int32_t* err, cudaStream_t s) {
  using C = TcCfg<R, BN>;
  CUtensorMap mh, ml, mk, mv;
  if (!encode_act_map(&mh, pa.xhi, pa.M, pa.E) || !encode_act_map(&ml, pa.xlo, pa.M, pa.E) ||
      !encode_weight_map(&mk, A_k, pa.H, pa.E, R, C::NG) || !encode_weight_map(&mv, A_v, pa.H, pa.E, R, C::NG))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(prefill_tc_kernel<R, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  TcArgs ta{};
  ta.M = pa.M; ta.T = pa.T; ta.H = pa.H; ta.bits = pa.bits; ta.L_cap = pa.L_cap; ta.KT = pa.E / kTcBK;
  ta.inv_p = pa.inv_p; ta.seq_lens = pa.seq_lens;
  ta.lat_k = pa.lat_k; ta.lat_v = pa.lat_v; ta.scale_k = pa.scale_k; ta.scale_v = pa.scale_v; ta.err = err;
  const dim3 grid((unsigned)((pa.M + kTcBM - 1) / kTcBM), (unsigned)(pa.N / C::BN));
  (void)cudaGetLastError();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_tc_kernel<R, BN>, mh, ml, mk, mv, ta);
}

// Output tile width of the tcgen05 path: 128 columns when the tiles hold whole
// heads of one side and there are enough of them to fill the device (every
// tile re-reads the activation rows of its m-tile from L2, so wider tiles
// halve that traffic); otherwise 64 (r <= 64), or 0 when the path does not
// apply.
int tc_tile_width(long long M, int H, int r) {
  if (r != 16 && r != 32 && r != 64 && r != 128) return 0;
  const long long hr = (long long)H * r, mt = (M + kTcBM - 1) / kTcBM;
  if (hr % 128 == 0 && (r == 128 || mt * (2 * hr / 128) >= 64)) return 128;
  if (r <= 64 && hr % 64 == 0) return 64;
  return 0;
}

// ------------------------------------------------------------------ 3. lengths
__global__ void prefill_advance_kernel(int32_t* seq_lens, int B, int T, int L_cap, int32_t* err) {
  griddep_wait();  // launched as a programmatic dependent of the GEMM, which reads the lengths
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int pos = seq_lens[b];
    if (pos >= 0 && (long long)pos + T <= L_cap) seq_lens[b] = pos + T;
    else set_err(err, WSVD_DEVERR_CACHE_FULL);
  }
}

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace wsvd

extern "C" size_t wsvd_prefill_workspace_size(int B, int T, int E) {
  if (B < 1 || T < 1 || E < 1) return 0;
  const size_t M = (size_t)B * T;
  return 2 * wsvd::align16(M * E * 2) + wsvd::align16(M * 4);
}

extern "C" int wsvd_latent_prefill(int B, int T, int H, int E, int r, int bits, int L_cap, int hadamard_block,
                                   const void* x, int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens,
                                   uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, void* workspace,
                                   size_t workspace_bytes, int32_t* err, void* stream) {
  using namespace wsvd;
  if (B < 0 || T < 0 || H < 1 || E < 1 || r < 1 || L_cap < 0) return WSVD_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return WSVD_OK;
  if (bits != 8 && bits != 4) return WSVD_ERR_INVALID_ARG;
  if (x_dtype != WSVD_DTYPE_FP16 && x_dtype != WSVD_DTYPE_BF16) return WSVD_ERR_INVALID_ARG;
  if (hadamard_block < 1 || hadamard_block > 1024 || (hadamard_block & (hadamard_block - 1)))
    return WSVD_ERR_INVALID_ARG;
  if (E % hadamard_block) return WSVD_ERR_INVALID_ARG;
  if (r % 8 || 128 % r || E % kBK || E > 16384) return WSVD_ERR_UNSUPPORTED;
  const long long M = (long long)B * T, N = 2LL * H * r;
  if (M > (1LL << 30) || (M + kBM - 1) / kBM > 0x7fffffffLL || (N + kBN - 1) / kBN > 65535) return WSVD_ERR_UNSUPPORTED;
  if (!x || !A_k || !A_v || !seq_lens || !lat_k || !lat_v || !scale_k || !scale_v || !workspace)
    return WSVD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(A_k) || !aligned16(A_v) || !aligned16(lat_k) || !aligned16(lat_v) ||
      !aligned16(scale_k) || !aligned16(scale_v) || !aligned16(workspace))
    return WSVD_ERR_INVALID_ARG;
  if (workspace_bytes < wsvd_prefill_workspace_size(B, T, E)) return WSVD_ERR_WORKSPACE_TOO_SMALL;

  uint8_t* w = static_cast<uint8_t*>(workspace);
  const size_t xbytes = align16((size_t)M * E * 2);
  PrefillArgs a{};
  a.B = B; a.T = T; a.M = (int)M; a.H = H; a.E = E; a.r = r; a.bits = bits; a.L_cap = L_cap; a.N = (int)N;
  a.xhi = reinterpret_cast<const __half*>(w);
  a.xlo = reinterpret_cast<const __half*>(w + xbytes);
  a.inv_p = reinterpret_cast<const float*>(w + 2 * xbytes);
  a.Ak = static_cast<const __half*>(A_k);
  a.Av = static_cast<const __half*>(A_v);
  a.seq_lens = seq_lens;
  a.lat_k = lat_k; a.lat_v = lat_v;
  a.scale_k = static_cast<__half*>(scale_k); a.scale_v = static_cast<__half*>(scale_v);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();  // the status below is these launches', not an earlier call's
  const size_t rot_smem = (size_t)E * 4;
  if (cudaFuncSetAttribute(prefill_rotate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rot_smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(prefill_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem) !=
          cudaSuccess)
    return WSVD_ERR_CUDA;
  const float hnorm = (float)(1.0 / sqrt((double)hadamard_block));
  __half* whi = reinterpret_cast<__half*>(w);
  __half* wlo = reinterpret_cast<__half*>(w + xbytes);
  float* winv = reinterpret_cast<float*>(w + 2 * xbytes);
  // Register path: the most threads per row (512, 256 or 128) that leave each
  // a power-of-two run of 4 .. 64 values and a block within a warp's reach.
  int nt = 0, ept = 0;
  for (int cand = 512; cand >= 128 && !nt; cand >>= 1) {
    const int e = E / cand;
    if (E % cand == 0 && e >= 4 && e <= 64 && (e & (e - 1)) == 0 && hadamard_block <= 32 * e) {
      nt = cand;
      ept = e;
    }
  }
  if (nt) {
#define WSVD_ROT(EPT_, NT_)                                                                                   \
  if (ept == EPT_ && nt == NT_)                                                                               \
    prefill_rotate_reg_kernel<EPT_, NT_><<<(unsigned)M, NT_, 0, s>>>(x, x_dtype, E, hadamard_block, hnorm, whi, \
                                                                    wlo, winv);
    WSVD_ROT(4, 128) WSVD_ROT(8, 128) WSVD_ROT(16, 128) WSVD_ROT(32, 128) WSVD_ROT(64, 128)
    WSVD_ROT(4, 256) WSVD_ROT(8, 256) WSVD_ROT(16, 256) WSVD_ROT(32, 256) WSVD_ROT(64, 256)
    WSVD_ROT(4, 512) WSVD_ROT(8, 512) WSVD_ROT(16, 512) WSVD_ROT(32, 512) WSVD_ROT(64, 512)
#undef WSVD_ROT
  } else {
    prefill_rotate_kernel<<<(unsigned)M, kRotThreads, rot_smem, s>>>(x, x_dtype, E, hadamard_block, hnorm, whi, wlo,
                                                                     winv);
  }
  const int bn = tc_tile_width(M, H, r);
  if (bn) {
    cudaError_t e = cudaSuccess;
    if (bn == 128) {
      switch (r) {
        case 16: e = launch_tc<16, 128>(a, A_k, A_v, err, s); break;
        case 32: e = launch_tc<32, 128>(a, A_k, A_v, err, s); break;
        case 64: e = launch_tc<64, 128>(a, A_k, A_v, err, s); break;
        default: e = launch_tc<128, 128>(a, A_k, A_v, err, s); break;
      }
    } else {
      switch (r) {
        case 16: e = launch_tc<16, 64>(a, A_k, A_v, err, s); break;
        case 32: e = launch_tc<32, 64>(a, A_k, A_v, err, s); break;
        default: e = launch_tc<64, 64>(a, A_k, A_v, err, s); break;
      }
    }
    if (e != cudaSuccess) return WSVD_ERR_CUDA;
  } else {
    const dim3 grid((unsigned)((M + kBM - 1) / kBM), (unsigned)((N + kBN - 1) / kBN));
    prefill_gemm_kernel<<<grid, kGemmThreads, kGemmSmem, s>>>(a);
  }
  {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, prefill_advance_kernel, seq_lens, B, T, L_cap, err) != cudaSuccess)
      return WSVD_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? WSVD_OK : WSVD_ERR_CUDA;
}
