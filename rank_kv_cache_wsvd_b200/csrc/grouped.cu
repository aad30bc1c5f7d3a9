// Grouped-query and multi-token decode over the per-head low-rank cache, on
// the sm_100a tensor cores (tcgen05, accumulators in tensor memory).
//
// The WSVD summaries describe one query per latent head and token (Japanese
// §2.4 "システム実装：融合カーネル", German §2.D: the fused low-rank
// flash-decoding kernel).  When several queries read the same latent head --
// G query heads sharing it (grouped-query attention) and/or Tq new tokens
// decoded at once -- one tile of cached latents serves all of them, and the
// two per-token products become dense contractions:
//     S[t][q]  = code_K[t] . q'_q            (tokens x queries, K = r)
//     O[j][q] += sum_t code_V[t][j] P~[t][q]  (latent dims x queries, K = tokens)
// with q'_q = B_Kh . q_q (reassociated as in the single-query kernel) and
// out_q = (O[:, q] / l_q) . B_Vh.
//
// Scores: q'_q is held as a 24-bit fixed-point integer in three SIGNED byte
// planes (x = h 2^16 + m 2^8 + l, each digit in [-127, 127]), so S is one
// kind::i8 product of the int8 codes (int4 codes widened to int8) with the
// 3 x queries plane rows: exact integer sums, combined once in fp32.
// Values: P~[t][q] = p_tq s_V,t 2^e_tile (a per-tile power of two keeps it in
// the fp16 normal range) split into fp16 hi + lo halves (22 significant
// bits); the codes are exact in fp16; one kind::f16 product per tile gives
// both halves as separate columns of the accumulator.
//
// Per CTA (one (b, latent head, query chunk) and one run of 128-token tiles):
//   warps 0-7  consumers, two warpgroups each holding half of the queries;
//              thread t of a group <-> token t of a tile <-> tensor-memory
//              lane t: widen the staged tile into the MMA operand layouts
//              (group 0 the K codes, group 1 the V codes), read the scores,
//              online softmax (exact per-tile maximum per query), write P~,
//              and fold each tile's O into registers;
//   warp 8     producer: 1-D bulk copies (TMA, no multicast) of codes + scales
//              into an mbarrier ring;
//   warp 9     allocates tensor memory and issues the MMAs (converged warp,
//              one elected lane).
// Split partials (m, l, O) merge last-arriver in split order (deterministic).
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "tc05.cuh"

namespace wsvd {
namespace {

constexpr int kGTok = 128;                    // tokens per tile (M of the score product)
constexpr int kGConsumers = 256;              // two consumer warpgroups (each half of the queries)
constexpr int kGThreads = kGConsumers + 64;   // + producer warp + MMA warp
constexpr int kGProducerWarp = 8, kGMmaWarp = 9;
constexpr int kMaxGroupedSplits = 64;
constexpr int kQMax = 8355711;                // 127 (2^16 + 2^8 + 1): largest 3-digit signed value

struct GroupedArgs {
  int B, Tq, Hq, Hkv, G, Hd, L_cap;
  int nqc;          // query chunks per (b, latent head)
  int nsplit;       // CTAs per (b, latent head, chunk)
  int chunk_tiles;  // tiles per split
  int slot_stride;  // partial slots per (b, latent head, chunk)
  const int32_t* seq_lens;
  const void* q;    // [B][Tq][Hq][Hd]
  int q_dtype;
  const uint8_t* lat_k;  // [B][Hkv][L_cap][RB]
  const uint8_t* lat_v;
  const __half* scale_k;  // [B][Hkv][L_cap]
  const __half* scale_v;
  const __half* Bk;  // [Hkv][r][Hd]
  const __half* Bv;
  float qscale;      // softmax_scale * log2 e
  float* out;        // [B][Tq][Hq][Hd]
  const uint8_t* qplanes;  // [B * Hkv * nqc] blocks of the q' planes (score operand layout) + steps
  float* partials;   // [B * Hkv * nqc][slot_stride][NQ][r + 2]
  int32_t* counters; // [B * Hkv * nqc], zero between calls
  int32_t* err;
};

template <int CODEC, int RB, int NQ>
struct GCfg {
  static constexpr int kBits = CODEC == kCodecI8 ? 8 : 4;
  static constexpr int R = RB * 8 / kBits;                 // latent rank
  static constexpr int KB = R < 32 ? 32 : R;               // int8 bytes per token of the score operand (K >= 32)
  static constexpr int KS = KB / 32;                       // score MMAs per tile
  static constexpr int MO = R <= 64 ? 64 : 128;            // M of the value product (latent rows, padded)
  static constexpr int NGRAN = MO == 64 ? 8 : 16;
  static constexpr int NS = (3 * NQ + 15) / 16 * 16;       // score columns: three planes per query
  static constexpr int NO = (2 * NQ + NGRAN - 1) / NGRAN * NGRAN;  // value columns: hi and lo per query
  static constexpr int NV = 3;  // value operand / P~ / value accumulator buffers (tile i folded two tiles later)
  static constexpr int TRAW = 2 * NS + NV * NO;
  static constexpr int TCOLS = TRAW <= 32 ? 32 : TRAW <= 64 ? 64 : TRAW <= 128 ? 128 : TRAW <= 256 ? 256 : 512;
  // shared memory, bytes
  static constexpr int STAGE = 2 * kGTok * RB + 2 * kGTok * 2;   // K codes, V codes, K scales, V scales
  static constexpr int S = STAGE <= 9216 ? 4 : 3;
  static constexpr int AK = kGTok * KB;                          // K-major int8: chunk c at c * 2048
  static constexpr int LBO_A = kGTok * 16;
  static constexpr int LBO_V = R * 16;                           // MN-major fp16: 8-token groups
  static constexpr int VC = (kGTok * R * 2 + 16 * (MO - R) + 127) / 128 * 128;  // + rows MO > R read past the end
  static constexpr int LBO_P = NO * 16;
  static constexpr int PB = kGTok * NO * 2;
  static constexpr int LBO_PL = NS * 16;
  static constexpr int PL = NS * KB;
  static constexpr int QBLOCK = PL + NQ * 4;                     // per query group: planes, then steps
  static constexpr int OFF_AK = S * STAGE;
  static constexpr int OFF_VC = OFF_AK + 2 * AK;
  static constexpr int OFF_P = OFF_VC + NV * VC;
  static constexpr int OFF_PL = OFF_P + NV * PB;
  static constexpr int OFF_STEP = OFF_PL + PL;                   // float step[NQ] (staged with the planes)
  static constexpr int OFF_WMAX = OFF_STEP + 2 * NQ * 4;         // float wmax[2][4][NQ]
  static constexpr int OFF_WSV = OFF_WMAX + 2 * 4 * NQ * 4;      // uint32 wsv[2][4]
  static constexpr int OFF_LSUM = OFF_WSV + 8 * 4;               // float lsum[4][NQ]
  static constexpr int OFF_BC = OFF_LSUM + 4 * NQ * 4;           // float2 bc[3][NQ] (new maximum, rescale)
  static constexpr int OFF_MRUN = OFF_BC + 3 * NQ * 8;            // float mrun[NQ], int be[3]
  static constexpr int OFF_RES = OFF_MRUN + NQ * 4 + 16;          // float res[NQ][R + 2]
  static constexpr int OFF_MISC = OFF_RES + NQ * (R + 2) * 4;    // int flag, uint32 tmem base
  static constexpr int OFF_BAR = (OFF_MISC + 16 + 7) / 8 * 8;
  static constexpr int NBAR = 2 * S + 11;
  static constexpr int SMEM_USED = OFF_BAR + NBAR * 8;
  // Shared memory requested at launch: at least enough that no more CTAs are
  // resident on an SM than its 512 tensor-memory columns can serve at once
  // (a CTA beyond that would wait inside its allocation).
  static constexpr int TMEM_CTAS = 512 / TCOLS;
  static constexpr int SMEM_FLOOR = 232448 / (TMEM_CTAS + 1) + 1;
  static constexpr int SMEM = SMEM_USED > SMEM_FLOOR ? SMEM_USED : SMEM_FLOOR;
  static_assert(RB % 16 == 0, "codes rows are whole 16-byte chunks");
  static_assert(NS <= 256 && NO <= 256, "MMA N");
};

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

// Two int8 codes (bytes `lo_sel`, `hi_sel` of the sign-flipped word x ^ 0x80808080)
// -> two exact fp16 values: the byte c + 128 lands in the mantissa of 1024.
__device__ __forceinline__ uint32_t i8pair_to_h2(uint32_t xflip, uint32_t sel) {
  const uint32_t w = __byte_perm(xflip, 0x64646464u, sel);
  __half2 h = *reinterpret_cast<const __half2*>(&w);
  h = __hsub2(h, __halves2half2(__float2half_rn(1152.f), __float2half_rn(1152.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

// 16 int8 codes -> 16 fp16 values (two 16-byte chunks).
__device__ __forceinline__ void i8x16_to_h(uint4 v, uint4& h0, uint4& h1) {
  const uint32_t x[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[2 * k] = i8pair_to_h2(x[k], 0x7140u);      // bytes 0, 1 -> low halves of two fp16 words
    o[2 * k + 1] = i8pair_to_h2(x[k], 0x7342u);  // bytes 2, 3
  }
  h0 = make_uint4(o[0], o[1], o[2], o[3]);
  h1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8 int4 codes of one word (element k in bits 4k..4k+3) -> 8 int8 bytes.
__device__ __forceinline__ uint2 i4x8_to_i8(uint32_t w) {
  const uint32_t ev = ((w & 0x0F0F0F0Fu) ^ 0x08080808u);         // c + 8 of elements 0, 2, 4, 6
  const uint32_t od = (((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u);  // c + 8 of elements 1, 3, 5, 7
  const uint32_t a = __byte_perm(ev, od, 0x5140u);  // elements 0, 1, 2, 3
  const uint32_t b = __byte_perm(ev, od, 0x7362u);  // elements 4, 5, 6, 7
  return make_uint2(__vsub4(a, 0x08080808u), __vsub4(b, 0x08080808u));
}

// 8 int4 codes of one word -> 8 exact fp16 values (one 16-byte chunk).
__device__ __forceinline__ uint4 i4x8_to_h(uint32_t w) {
  const uint32_t ev = ((w & 0x0F0F0F0Fu) ^ 0x08080808u);
  const uint32_t od = (((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u);
  uint32_t o[4];
  const __half2 off = __halves2half2(__float2half_rn(1032.f), __float2half_rn(1032.f));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // byte 0 <- element 2k (ev byte k), byte 2 <- element 2k + 1 (od byte k)
    const uint32_t u = __byte_perm(ev, od, (uint32_t)k | ((uint32_t)(4 + k) << 8)) & 0x00FF00FFu;
    const uint32_t hw = u | 0x64006400u;  // (c + 8) in the mantissa of 1024
    __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&hw), off);
    o[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Stores N fp16 values (N / 2 packed pairs) at columns c0 .. c0 + N - 1 of a
// row whose 8-column core-matrix chunks lie 128 bytes apart (c0 a multiple of N).
template <int N>
__device__ __forceinline__ void store_cols(uint32_t row, int c0, const uint32_t (&w)[N / 2]) {
  const uint32_t a = row + (uint32_t)((c0 >> 3) * 128 + (c0 & 7) * 2);
  if constexpr (N == 8) {
    sts128(a, make_uint4(w[0], w[1], w[2], w[3]));
  } else if constexpr (N == 4) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(w[0]), "r"(w[1]) : "memory");
  } else {
    static_assert(N == 2, "query counts per group: 2, 4 or 8");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(w[0]) : "memory");
  }
}

// An integer below 2^22 in magnitude to fp32, exactly, on the FMA pipe:
// adding it to the bits of 1.5 * 2^23 lands it in that float's mantissa.
__device__ __forceinline__ float small_int_to_f32(uint32_t v) {
  return __int_as_float((int)v + 0x4B400000) - 12582912.f;
}

// Score of query q from its three plane sums (h 2^16 + m 2^8 + l); every plane
// sum is below 128 * 127 * 127 < 2^21 in magnitude.
template <int N>
__device__ __forceinline__ float plane_sum(const uint32_t (&sv)[N], int q) {
  return fmaf(small_int_to_f32(sv[3 * q]), 65536.f,
              fmaf(small_int_to_f32(sv[3 * q + 1]), 256.f, small_int_to_f32(sv[3 * q + 2])));
}

// q' of every query of one (b, latent head, query chunk) group, as the score
// operand the decode kernel stages: q'_q = (B_Kh . q_q) * softmax_scale * log2 e,
// quantised with step max|q'_q| / 8355711 and written as three signed byte
// planes in the K-major no-swizzle layout, followed by the NQ steps.  One CTA
// per group: B_Kh and the group's query rows are first staged in shared memory
// with coalesced 16-byte loads; each output is then a dot product over the
// head dimension in a fixed (row-rotated) order.  The decode grid is launched
// behind this one as a programmatic dependent.
template <int CODEC, int RB, int NQ>
__global__ void __launch_bounds__(128) grouped_qproj_kernel(const GroupedArgs a, uint8_t* qplanes) {
  using C = GCfg<CODEC, RB, NQ>;
  constexpr int R = C::R, NS = C::NS;
  extern __shared__ __align__(16) uint8_t psm[];
  __half* bks = reinterpret_cast<__half*>(psm);                         // [R][Hd]
  float* qs = reinterpret_cast<float*>(psm + (size_t)R * a.Hd * 2);     // [NQ][Hd]
  float* qp = qs + (size_t)NQ * a.Hd;                                   // [NQ][R]
  float* inv = qp + NQ * R;                                             // [NQ]
  griddep_launch_dependents();
  const int grp = blockIdx.x, t = threadIdx.x;
  const int qc = grp % a.nqc, hkv = (grp / a.nqc) % a.Hkv, b = grp / (a.nqc * a.Hkv);
  const int nq = min(NQ, a.G * a.Tq - qc * NQ);
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.Bk + (size_t)hkv * R * a.Hd);
    uint4* dst = reinterpret_cast<uint4*>(bks);
    for (int i = t; i < R * a.Hd / 8; i += 128) dst[i] = src[i];
  }
  for (int i = t; i < NQ * a.Hd / 8; i += 128) {  // 8 query values per 16-byte load
    const int ql = i / (a.Hd / 8), k8 = i % (a.Hd / 8);
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (ql < nq) {
      const int qg = qc * NQ + ql, tq = qg / a.G, g = qg % a.G;
      w = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.q) +
                                         (((size_t)b * a.Tq + tq) * a.Hq + (size_t)hkv * a.G + g) * a.Hd)[k8];
    }
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint16_t h16 = (uint16_t)(u[c >> 1] >> (16 * (c & 1)));
      qs[ql * a.Hd + 8 * k8 + c] = a.q_dtype == WSVD_DTYPE_BF16 ? __uint_as_float((uint32_t)h16 << 16)
                                                                 : __half2float(__ushort_as_half(h16));
    }
  }
  __syncthreads();
  for (int o = t; o < NQ * R; o += 128) {
    const int ql = o / R, j = o % R;
    const __half* brow = bks + (size_t)j * a.Hd;
    const float* qrow = qs + (size_t)ql * a.Hd;
    float d = 0.f;
    for (int kk = 0; kk < a.Hd; ++kk) {
      const int k = (kk + j) & (a.Hd - 1);  // rows start at different columns: distinct banks
      d = fmaf(__half2float(brow[k]), qrow[k], d);
    }
    qp[o] = d * a.qscale;
  }
  __syncthreads();
  uint8_t* blk = qplanes + (size_t)grp * C::QBLOCK;
  float* steps = reinterpret_cast<float*>(blk + C::PL);
  if (t < NQ) {
    float m = 0.f;
    for (int j = 0; j < R; ++j) m = fmaxf(m, fabsf(qp[t * R + j]));
    steps[t] = m > 0.f ? m / (float)kQMax : 0.f;
    inv[t] = m > 0.f ? (float)kQMax / m : 0.f;
  }
  __syncthreads();
  for (int idx = t; idx < NS * C::KB; idx += 128) {
    const int n = idx / C::KB, k = idx % C::KB;
    int dig = 0;
    if (n < 3 * NQ && k < R) {
      const int ql = n / 3, p = n % 3;
      const int x = max(-kQMax, min(kQMax, __float2int_rn(qp[ql * R + k] * inv[ql])));
      const int l0 = ((x + 128) & 255) - 128, x1 = (x - l0) >> 8;
      const int m0 = ((x1 + 128) & 255) - 128, h0 = (x1 - m0) >> 8;
      dig = p == 0 ? h0 : (p == 1 ? m0 : l0);
    }
    blk[(k >> 4) * C::LBO_PL + (n >> 3) * 128 + (n & 7) * 16 + (k & 15)] = (uint8_t)(int8_t)dig;
  }
}

__host__ inline size_t qproj_smem_bytes(int R, int NQ, int Hd) {
  return (size_t)R * Hd * 2 + (size_t)NQ * Hd * 4 + (size_t)NQ * R * 4 + (size_t)NQ * 4;
}

template <int CODEC, int RB, int NQ>
__global__ void __launch_bounds__(kGThreads, 2) grouped_decode_kernel(const GroupedArgs a) {
  using C = GCfg<CODEC, RB, NQ>;
  constexpr int R = C::R, S = C::S, NS = C::NS, NO = C::NO, MO = C::MO;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, qc = (int)(blockIdx.y % a.nqc), hkv = (int)(blockIdx.y / a.nqc), b = blockIdx.z;
  const int nq_group = a.G * a.Tq;
  const int nq = min(NQ, nq_group - qc * NQ);  // real queries of this CTA

  const int raw = a.seq_lens[b];
  const bool bad = raw < 0 || raw > a.L_cap;
  if (bad && split == 0 && hkv == 0 && qc == 0 && tid == 0) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
  const int len = bad ? 0 : raw;
  const int span = a.chunk_tiles * kGTok;
  const int ncontrib = (len + span - 1) / span;
  auto out_row = [&](int ql) {  // output row of local query ql
    const int qg = qc * NQ + ql, tq = qg / a.G, g = qg % a.G;
    return a.out + (((size_t)b * a.Tq + tq) * a.Hq + (size_t)hkv * a.G + g) * a.Hd;
  };
  if (split >= ncontrib) {  // no cached token for this CTA (uniform exit before any set-up)
    if (split == 0)
      for (int i = tid; i < nq * a.Hd; i += kGThreads) out_row(i / a.Hd)[i % a.Hd] = 0.f;
    griddep_wait();  // the grid never completes before the projection grid it was launched behind
    return;
  }
  const int t_begin = split * span;
  const int t_end = min(len, t_begin + span);
  const int ntiles = (t_end - t_begin + kGTok - 1) / kGTok;
  const size_t head_row = ((size_t)b * a.Hkv + hkv) * a.L_cap;

  uint8_t* ring = smem;
  const uint32_t s_ak = smem_u32(smem + C::OFF_AK), s_vc = smem_u32(smem + C::OFF_VC);
  const uint32_t s_p = smem_u32(smem + C::OFF_P), s_pl = smem_u32(smem + C::OFF_PL);
  float* stepv = reinterpret_cast<float*>(smem + C::OFF_STEP);
  float* wmax = reinterpret_cast<float*>(smem + C::OFF_WMAX);
  uint32_t* wsv = reinterpret_cast<uint32_t*>(smem + C::OFF_WSV);
  float* lsum = reinterpret_cast<float*>(smem + C::OFF_LSUM);
  float* res = reinterpret_cast<float*>(smem + C::OFF_RES);
  float2* bc = reinterpret_cast<float2*>(smem + C::OFF_BC);  // per tile parity: each query's new maximum, rescale
  float* mrun = reinterpret_cast<float*>(smem + C::OFF_MRUN); // running maximum per query
  int* be = reinterpret_cast<int*>(smem + C::OFF_MRUN + NQ * 4); // per tile parity: the P~ exponent
  int* flag = reinterpret_cast<int*>(smem + C::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + S;
  constexpr int NV = C::NV;
  uint64_t* conv = empty + S;   // [2] tile operands widened (128 arrivals)
  uint64_t* sready = conv + 2;  // [2] score MMAs done (commit)
  uint64_t* pfull = sready + 2; // [NV] P~ written (128 arrivals)
  uint64_t* oready = pfull + NV; // [NV] value MMAs done (commit)
  uint64_t* pready = oready + NV; // the group's q' planes and steps are staged

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGConsumers / 32);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&conv[s], kGConsumers);
      mbar_init(&sready[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&pfull[s], kGConsumers);
      mbar_init(&oready[s], 1);
    }
    mbar_init(pready, 1);
    fence_mbar_init();
  }
  if (warp == kGMmaWarp) tc05::alloc(tmem_slot, C::TCOLS);
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

  // The producer and MMA warps run their loops converged (every lane waits,
  // one elected lane issues), so that copies and MMAs issue at full rate.
  if (warp == kGProducerWarp) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_evict_first_policy();
    const int gidx = (b * a.Hkv + hkv) * a.nqc + qc;
    {  // warm B_Vh in L2 for whichever split finishes the group (read at the very end)
      const char* bv = reinterpret_cast<const char*>(a.Bv + (size_t)hkv * R * a.Hd);
      const int bytes = R * a.Hd * 2;
      for (int o = lane * 128; o < bytes; o += 32 * 128) prefetch_l2(bv + o);
    }
    auto stage_planes = [&]() {  // the q' planes and steps (written by the preceding grid)
      griddep_wait();
      mbar_arrive_expect_tx_warp(pready, (uint32_t)C::QBLOCK);
      bulk_g2s_warp(smem + C::OFF_PL, a.qplanes + (size_t)gidx * C::QBLOCK, (uint32_t)C::PL, pready,
                    l2_evict_last_policy());
      bulk_g2s_warp(smem + C::OFF_STEP, a.qplanes + (size_t)gidx * C::QBLOCK + C::PL, (uint32_t)(NQ * 4), pready,
                    l2_evict_last_policy());
    };
    for (int i = 0; i < ntiles; ++i) {
      if (i == min(S, ntiles)) stage_planes();  // the ring is primed: now the planes
      const int s = i % S;
      if (i >= S) wait(&empty[s], (uint32_t)(((i / S) - 1) & 1));
      __syncwarp();
      const int r0 = t_begin + i * kGTok, n = min(kGTok, t_end - r0);
      const uint32_t cb = (uint32_t)n * RB, sb = (uint32_t)((n + 7) & ~7) * 2u;
      uint8_t* st = ring + (size_t)s * C::STAGE;
      mbar_arrive_expect_tx_warp(&full[s], 2 * cb + 2 * sb);
      bulk_g2s_warp(st, a.lat_k + (head_row + r0) * RB, cb, &full[s], pol);
      bulk_g2s_warp(st + kGTok * RB, a.lat_v + (head_row + r0) * RB, cb, &full[s], pol);
      bulk_g2s_warp(st + 2 * kGTok * RB, a.scale_k + head_row + r0, sb, &full[s], pol);
      bulk_g2s_warp(st + 2 * kGTok * RB + 2 * kGTok, a.scale_v + head_row + r0, sb, &full[s], pol);
    }
    if (ntiles <= S) stage_planes();  // fewer tiles than stages: the planes follow the last tile
    // no copy left in flight: the last uses of every stage and the planes have landed
    for (int i = max(0, ntiles - S); i < ntiles; ++i) wait(&full[i % S], (uint32_t)((i / S) & 1));
    wait(pready, 0);
    __syncwarp();
  } else if (warp == kGMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = tc05::instr_desc(2, 1, 1, 0, 0, kGTok, NS);
    constexpr uint32_t idesc_o = tc05::instr_desc(1, 0, 0, 1, 1, MO, NO);
    auto scores = [&](int j) {
      wait(&conv[j & 1], (uint32_t)((j >> 1) & 1));
      __syncwarp();
      tc05::fence_after_sync();
      const uint32_t d = tmem + (uint32_t)((j & 1) * NS);
      const uint32_t abase = s_ak + (uint32_t)((j & 1) * C::AK);
#pragma unroll
      for (int kk = 0; kk < C::KS; ++kk)
        tc05::mma_i8_warp(d, tc05::smem_desc(abase + kk * 2 * C::LBO_A, C::LBO_A, 128),
                          tc05::smem_desc(s_pl + kk * 2 * C::LBO_PL, C::LBO_PL, 128), idesc_s, kk > 0);
      tc05::commit_warp(&sready[j & 1]);
    };
    wait(pready, 0);  // the q' planes (score operand B) are staged
    scores(0);
    for (int i = 0; i < ntiles; ++i) {
      if (i + 1 < ntiles) scores(i + 1);
      const int vb = i % NV;
      wait(&pfull[vb], (uint32_t)((i / NV) & 1));
      __syncwarp();
      tc05::fence_after_sync();
      const uint32_t d = tmem + (uint32_t)(2 * NS + vb * NO);
      const uint32_t vbase = s_vc + (uint32_t)(vb * C::VC), pbase = s_p + (uint32_t)(vb * C::PB);
#pragma unroll
      for (int kk = 0; kk < kGTok / 16; ++kk)
        tc05::mma_f16_warp(d, tc05::smem_desc(vbase + kk * 2 * C::LBO_V, C::LBO_V, 128),
                           tc05::smem_desc(pbase + kk * 2 * C::LBO_P, C::LBO_P, 128), idesc_o, kk > 0);
      tc05::commit_warp(&oready[vb]);
    }
    // every MMA has completed before the allocation is released
    wait(&oready[(ntiles - 1) % NV], (uint32_t)(((ntiles - 1) / NV) & 1));
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    // Two warpgroups: thread ct of 256 is token slot t = ct % 128 of the tile
    // (tensor-memory lane t, warp quarter wq = warp % 4) for the queries of its
    // group, q0 .. q0 + NQH - 1.  Group 0 widens the K codes of a staged tile,
    // group 1 the V codes.
    constexpr int NQH = NQ / 2;
    const int ct = tid, grp = tid >> 7, t = tid & 127, wq = warp & 3, q0 = grp * NQH;
    wait(pready, 0);  // the group's steps (and planes) are staged
    float step[NQH];
    int nvis[NQH];  // rows visible to each of this thread's queries
    const int vis_min = len - a.Tq + 1 + (qc * NQ) / a.G;  // the chunk's first query sees the fewest
#pragma unroll
    for (int q = 0; q < NQH; ++q) {
      const int qg = q0 + q;
      step[q] = stepv[qg];
      const int tq = (qc * NQ + qg) / a.G;
      nvis[q] = qg < nq ? len - a.Tq + 1 + tq : 0;
    }

    // Widen tile j of the ring into the operand buffers (K codes: slot j & 1,
    // group 0; V codes: slot j % NV, group 1).
    auto convert = [&](int j, float& sk, float& sv, int& pos) {
      const int s = j % S;
      wait(&full[s], (uint32_t)((j / S) & 1));
      const uint8_t* st = ring + (size_t)s * C::STAGE;
      if (grp == 0) {
        const uint32_t ak = s_ak + (uint32_t)((j & 1) * C::AK) + (uint32_t)((t >> 3) * 128 + (t & 7) * 16);
        const uint32_t kr = smem_u32(st + t * RB);
#pragma unroll
        for (int c = 0; c < RB / 16; ++c) {
          const uint4 kv = lds128(kr + 16 * c);
          if constexpr (CODEC == kCodecI8) {
            sts128(ak + c * C::LBO_A, kv);
          } else {
            const uint2 k0 = i4x8_to_i8(kv.x), k1 = i4x8_to_i8(kv.y), k2 = i4x8_to_i8(kv.z), k3 = i4x8_to_i8(kv.w);
            sts128(ak + (2 * c) * C::LBO_A, make_uint4(k0.x, k0.y, k1.x, k1.y));
            sts128(ak + (2 * c + 1) * C::LBO_A, make_uint4(k2.x, k2.y, k3.x, k3.y));
          }
        }
      } else {
        const uint32_t vc = s_vc + (uint32_t)((j % NV) * C::VC) + (uint32_t)((t >> 3) * C::LBO_V + (t & 7) * 16);
        const uint32_t vr = smem_u32(st + kGTok * RB + t * RB);
#pragma unroll
        for (int c = 0; c < RB / 16; ++c) {
          const uint4 vv = lds128(vr + 16 * c);
          if constexpr (CODEC == kCodecI8) {
            uint4 h0, h1;
            i8x16_to_h(vv, h0, h1);
            sts128(vc + (2 * c) * 128, h0);
            sts128(vc + (2 * c + 1) * 128, h1);
          } else {
            sts128(vc + (4 * c) * 128, i4x8_to_h(vv.x));
            sts128(vc + (4 * c + 1) * 128, i4x8_to_h(vv.y));
            sts128(vc + (4 * c + 2) * 128, i4x8_to_h(vv.z));
            sts128(vc + (4 * c + 3) * 128, i4x8_to_h(vv.w));
          }
        }
      }
      sk = lds_half_as_float(smem_u32(st + 2 * kGTok * RB + 2 * t));
      sv = lds_half_as_float(smem_u32(st + 2 * kGTok * RB + 2 * kGTok + 2 * t));
      pos = t_begin + j * kGTok + t;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      tc05::fence_proxy_async_smem();
      mbar_arrive(&conv[j & 1]);
    };

    // Rows of the value accumulator this thread holds: M = 64 puts row j in
    // lane (j % 16) + 32 (j / 16), M = 128 row j in lane j.
    const int orow = MO == 64 ? (lane < 16 ? wq * 16 + lane : -1) : t;
    const bool holder = orow >= 0 && orow < R;
    const bool warp_holds = MO == 64 ? wq * 16 < R : wq * 32 < R;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    float l[NQH], acc[NQH];
#pragma unroll
    for (int q = 0; q < NQH; ++q) {
      l[q] = 0.f;
      acc[q] = 0.f;
    }
    if (ct < NQ) mrun[ct] = kNegInf;  // ordered before its first use by the tile barriers
    // Fold tile j's value accumulator (scaled by 2^-e_j) into acc, rescaled
    // from the maxima before tile j to the maxima after it (the factor tile
    // j's softmax step broadcast: 0 while nothing was seen, 1 while a query
    // still sees nothing, when its columns are zero).
    auto accumulate = [&](int j) {
      const int vb = j % NV;
      wait(&oready[vb], (uint32_t)((j / NV) & 1));
      tc05::fence_after_sync();
      if (warp_holds) {
        const int e = be[vb];
        constexpr int NL = (NQH + 7) / 8 * 8;
        uint32_t vh[NL], vl[NL];
        const uint32_t ta = lane_base + (uint32_t)(2 * NS + vb * NO + q0);
#pragma unroll
        for (int c = 0; c < NL / 8; ++c) {
          uint32_t w8[8];
          tc05::ld8(ta + 8 * c, w8);
#pragma unroll
          for (int k = 0; k < 8; ++k) vh[8 * c + k] = w8[k];
          tc05::ld8(ta + NQ + 8 * c, w8);
#pragma unroll
          for (int k = 0; k < 8; ++k) vl[8 * c + k] = w8[k];
        }
        tc05::wait_ld();
        const float unscale = __int_as_float((127 - e) << 23);
        const float2* bj = bc + vb * NQ + q0;
#pragma unroll
        for (int q = 0; q < NQH; ++q) {
          const float d = (__uint_as_float(vh[q]) + __uint_as_float(vl[q])) * unscale;
          acc[q] = fmaf(acc[q], bj[q].y, d);
        }
      }
      tc05::fence_before_sync();
    };

    float sk_cur, sv_cur;
    int pos_cur;
    convert(0, sk_cur, sv_cur, pos_cur);
    for (int i = 0; i < ntiles; ++i) {
      // tile i - 2's value product was issued a whole tile ago; its buffers
      // (value operand, P~, accumulator) are then free for tile i + 1
      if (i >= 2) accumulate(i - 2);
      float sk_n = 0.f, sv_n = 0.f;
      int pos_n = 0;
      if (i + 1 < ntiles) convert(i + 1, sk_n, sv_n, pos_n);
      // scores of tile i: this thread's queries' three plane sums
      wait(&sready[i & 1], (uint32_t)((i >> 1) & 1));
      tc05::fence_after_sync();
      constexpr int NSV = (3 * NQH + 7) / 8 * 8;
      uint32_t sv32[NSV];
      {
        const uint32_t ta = lane_base + (uint32_t)((i & 1) * NS + 3 * q0);
#pragma unroll
        for (int c = 0; c < NSV / 8; ++c) {
          uint32_t w8[8];
          tc05::ld8(ta + 8 * c, w8);
#pragma unroll
          for (int k = 0; k < 8; ++k) sv32[8 * c + k] = w8[k];
        }
        tc05::wait_ld();
      }
      float s[NQH];
      float* wm = wmax + (i & 1) * 4 * NQ;
      // Every row of a tile below the first query's horizon is visible to all
      // real queries: no per-query test there.
      if (nq == NQ && t_begin + (i + 1) * kGTok <= vis_min) {
#pragma unroll
        for (int q = 0; q < NQH; ++q) s[q] = plane_sum(sv32, q) * step[q] * sk_cur;
      } else {
#pragma unroll
        for (int q = 0; q < NQH; ++q) s[q] = pos_cur < nvis[q] ? plane_sum(sv32, q) * step[q] * sk_cur : kNegInf;
      }
#pragma unroll
      for (int q = 0; q < NQH; ++q) {
        const float mx = warp_max_f32(s[q]);
        if (lane == 0) wm[wq * NQ + q0 + q] = mx;
      }
      if (grp == 0) {
        const uint32_t svb = pos_cur < len ? (uint32_t)__half_as_ushort(__float2half_rn(sv_cur)) : 0u;
        const uint32_t svm = warp_max_u32(svb);
        if (lane == 0) wsv[(i & 1) * 4 + wq] = svm;
      }
      tc05::fence_before_sync();
      named_barrier_sync(1, kGConsumers);
      // One thread per query: the tile maximum over the four warp quarters, the
      // new running maximum and the rescale of the old one; one thread: the P~
      // scale 2^e that puts the largest s_V of the tile in [2^14, 2^15).
      float2* bi = bc + (i % NV) * NQ;
      if (ct < NQ) {
        float tmax = wm[ct];
#pragma unroll
        for (int w = 1; w < 4; ++w) tmax = fmaxf(tmax, wm[w * NQ + ct]);
        const float mold = mrun[ct], mnew = fmaxf(mold, tmax);
        // .x: the maximum the tile's exponentials are taken against (0 while
        // the query sees nothing, so that -inf - .x stays -inf); .y: rescale
        bi[ct] = make_float2(mnew == kNegInf ? 0.f : mnew, mnew == kNegInf ? 1.f : ex2(mold - mnew));
        mrun[ct] = mnew;
      } else if (ct == kGConsumers - 1) {
        uint32_t svmax = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) svmax = max(svmax, wsv[(i & 1) * 4 + w]);
        const float svmf = __half2float(__ushort_as_half((uint16_t)svmax));
        be[i % NV] = svmf > 0.f ? 14 - (((__float_as_int(svmf) >> 23) & 0xFF) - 127) : 0;
      }
      named_barrier_sync(1, kGConsumers);
      const int e = be[i % NV];
      const float svs = (pos_cur < len) ? sv_cur * __int_as_float((127 + e) << 23) : 0.f;
      uint32_t ph[NQH / 2], pl[NQH / 2];  // fp16 pairs of this group's hi and lo P~ columns
#pragma unroll
      for (int q = 0; q < NQH; q += 2) {
        const float2 m0 = bi[q0 + q], m1 = bi[q0 + q + 1];
        const float p0 = ex2(s[q] - m0.x), p1 = ex2(s[q + 1] - m1.x);  // 0 for a row the query does not see
        l[q] = fmaf(l[q], m0.y, p0);
        l[q + 1] = fmaf(l[q + 1], m1.y, p1);
        const float t0 = p0 * svs, t1 = p1 * svs;
        const __half2 hi = __floats2half2_rn(t0, t1);
        const float2 hf = __half22float2(hi);
        const __half2 lo = __floats2half2_rn(t0 - hf.x, t1 - hf.y);
        ph[q >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
        pl[q >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      // P~ row of token t: column c at byte (c / 8) * 128 + (c % 8) * 2 of the row's core-matrix run
      const uint32_t pa = s_p + (uint32_t)((i % NV) * C::PB) + (uint32_t)((t >> 3) * C::LBO_P + (t & 7) * 16);
      store_cols<NQH>(pa, q0, ph);
      store_cols<NQH>(pa, NQ + q0, pl);
      if (grp == 1) {
#pragma unroll
        for (int c = 2 * NQ / 8; c < NO / 8; ++c) sts128(pa + c * 128, make_uint4(0u, 0u, 0u, 0u));
      }
      tc05::fence_proxy_async_smem();
      mbar_arrive(&pfull[i % NV]);
      sk_cur = sk_n;
      sv_cur = sv_n;
      pos_cur = pos_n;
    }
    for (int j = max(0, ntiles - 2); j < ntiles; ++j) accumulate(j);

    // CTA partial per query: (m, l, O[R])
#pragma unroll
    for (int q = 0; q < NQH; ++q) {
      float v = l[q];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) lsum[wq * NQ + q0 + q] = v;
    }
    if (holder)
#pragma unroll
      for (int q = 0; q < NQH; ++q) res[(q0 + q) * (R + 2) + 2 + orow] = acc[q];
    named_barrier_sync(1, kGConsumers);
    if (ct < NQ) {
      res[ct * (R + 2)] = mrun[ct];
      res[ct * (R + 2) + 1] = ((lsum[ct] + lsum[NQ + ct]) + lsum[2 * NQ + ct]) + lsum[3 * NQ + ct];
    }
    named_barrier_sync(1, kGConsumers);

    const int gidx = (b * a.Hkv + hkv) * a.nqc + qc;
    const float* fin = res;
    bool finish = true;
    if (ncontrib > 1) {
      float* dst = a.partials + ((size_t)gidx * a.slot_stride + split) * NQ * (R + 2);
      for (int e2 = ct; e2 < nq * (R + 2); e2 += kGConsumers) dst[e2] = res[e2];
      __threadfence();
      named_barrier_sync(1, kGConsumers);
      if (ct == 0) flag[0] = atomicAdd(&a.counters[gidx], 1) == ncontrib - 1;
      named_barrier_sync(1, kGConsumers);
      finish = flag[0] != 0;
      if (finish) {  // last arriver: merge the splits in order
        __threadfence();
        const float* part = a.partials + (size_t)gidx * a.slot_stride * NQ * (R + 2);
        for (int e2 = ct; e2 < nq * (R + 1); e2 += kGConsumers) {
          const int ql = e2 / (R + 1), col = 1 + e2 % (R + 1);
          float M = kNegInf;
          for (int sp = 0; sp < ncontrib; ++sp) M = fmaxf(M, __ldcg(part + ((size_t)sp * NQ + ql) * (R + 2)));
          float acc2 = 0.f;
          for (int sp = 0; sp < ncontrib; ++sp) {
            const float mp = __ldcg(part + ((size_t)sp * NQ + ql) * (R + 2));
            if (mp != kNegInf) acc2 = fmaf(ex2(mp - M), __ldcg(part + ((size_t)sp * NQ + ql) * (R + 2) + col), acc2);
          }
          res[ql * (R + 2) + col] = acc2;
        }
        named_barrier_sync(1, kGConsumers);
        if (ct == 0) atomicExch(&a.counters[gidx], 0);
      }
    }
    if (finish) {  // out_q = (O_q / l_q) . B_Vh
      for (int idx = ct; idx < nq * a.Hd; idx += kGConsumers) {
        const int ql = idx / a.Hd, d = idx % a.Hd;
        const float* rq = fin + ql * (R + 2);
        const float inv = rq[1] > 0.f ? 1.f / rq[1] : 0.f;
        const __half* bv = a.Bv + (size_t)hkv * R * a.Hd + d;
        float sacc = 0.f;
        for (int j = 0; j < R; ++j) sacc = fmaf(rq[2 + j], __half2float(bv[(size_t)j * a.Hd]), sacc);
        out_row(ql)[d] = sacc * inv;
      }
    }
  }
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == kGMmaWarp) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, C::TCOLS);
  }
}

// ---------------------------------------------------------------- host side
int nq_per_cta(int nq_group) { return nq_group <= 4 ? 4 : (nq_group <= 8 ? 8 : 16); }

struct GroupedKernels {
  const void* qproj;   // grouped_qproj_kernel
  const void* decode;  // grouped_decode_kernel
  size_t smem;
  int tmem_ctas;       // CTAs per SM that the 512 tensor-memory columns serve at once
};

template <int CODEC, int RB, int NQ>
GroupedKernels kernels_of() {
  return GroupedKernels{reinterpret_cast<const void*>(&grouped_qproj_kernel<CODEC, RB, NQ>),
                        reinterpret_cast<const void*>(&grouped_decode_kernel<CODEC, RB, NQ>),
                        (size_t)GCfg<CODEC, RB, NQ>::SMEM, GCfg<CODEC, RB, NQ>::TMEM_CTAS};
}

template <int CODEC, int RB>
GroupedKernels pick_nq(int nq) {
  switch (nq) {
    case 4: return kernels_of<CODEC, RB, 4>();
    case 8: return kernels_of<CODEC, RB, 8>();
    default: return kernels_of<CODEC, RB, 16>();
  }
}

bool pick_grouped(int bits, int rb, int nq, GroupedKernels* k) {
  if (bits == 8) {
    if (rb == 16) { *k = pick_nq<kCodecI8, 16>(nq); return true; }
    if (rb == 32) { *k = pick_nq<kCodecI8, 32>(nq); return true; }
    if (rb == 64) { *k = pick_nq<kCodecI8, 64>(nq); return true; }
  } else {
    if (rb == 16) { *k = pick_nq<kCodecI4, 16>(nq); return true; }
    if (rb == 32) { *k = pick_nq<kCodecI4, 32>(nq); return true; }
    if (rb == 64) { *k = pick_nq<kCodecI4, 64>(nq); return true; }
  }
  return false;
}

std::mutex g_mu;
std::map<std::pair<const void*, int>, int> g_occ;  // (kernel, device) -> resident CTAs per SM (smem opted in)
std::map<int, int> g_sms;

// Opts the kernel into its shared memory and returns (SMs, resident CTAs per
// SM).  The residency is worked out from the kernel's registers, its shared
// memory and its tensor-memory columns (the occupancy query knows nothing of
// the last).
cudaError_t device_setup(const void* fn, size_t smem, int tmem_ctas, int* sms, int* occ) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(fn, dev);
  auto it = g_occ.find(key);
  if (it != g_occ.end()) {
    *occ = it->second;
    *sms = g_sms[dev];
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int n = 148, sm_smem = 233472, sm_regs = 65536, reserved = 1024;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaFuncAttributes fa{};
  int o = tmem_ctas;
  if (cudaFuncGetAttributes(&fa, fn) == cudaSuccess && fa.numRegs > 0) {
    const int warp_regs = (fa.numRegs * 32 + 255) / 256 * 256;  // allocated per warp in 256-register units
    o = std::min(o, sm_regs / (warp_regs * (kGThreads / 32)));
  }
  o = std::min(o, (int)(sm_smem / (smem + (size_t)reserved)));
  o = std::max(o, 1);
  g_occ[key] = o;
  g_sms[dev] = n;
  *occ = o;
  *sms = n;
  return cudaSuccess;
}

// Splits per (b, latent head, query chunk): as many as fill the resident CTA
// slots in one wave (a grid a little over a whole number of waves leaves a
// tail as long as a CTA), never more than there are tiles or partial slots.
int grouped_splits(long long groups, int tiles_cap, int slots, int sms, int occ) {
  const long long resident = (long long)sms * occ;
  const long long per_group = groups >= resident ? 1 : resident / groups;
  return (int)std::max<long long>(1, std::min<long long>(std::min<long long>(tiles_cap, slots), per_group));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

struct GroupedShape {
  int nq, nqc, slots;
  size_t partial_bytes, counter_bytes, plane_bytes, total;
};
GroupedShape grouped_shape(int B, int Tq, int Hq, int Hkv, int r, int L_cap) {
  GroupedShape s{};
  const int G = Hq / Hkv, nq_group = G * Tq;
  s.nq = nq_per_cta(nq_group);
  s.nqc = (nq_group + s.nq - 1) / s.nq;
  const int tiles_cap = std::max(1, (L_cap + kGTok - 1) / kGTok);
  s.slots = std::min(tiles_cap, kMaxGroupedSplits);
  s.partial_bytes = align16((size_t)B * Hkv * s.nqc * s.slots * s.nq * (r + 2) * sizeof(float));
  s.counter_bytes = align16((size_t)B * Hkv * s.nqc * 4);
  // q' planes per group: (3 nq rounded up to 16) rows of max(32, r) bytes, then nq fp32 steps
  const size_t qblock = (size_t)((3 * s.nq + 15) / 16 * 16) * (r < 32 ? 32 : r) + (size_t)s.nq * 4;
  s.plane_bytes = align16((size_t)B * Hkv * s.nqc * qblock);
  s.total = s.partial_bytes + s.counter_bytes + s.plane_bytes;
  return s;
}

}  // namespace
}  // namespace wsvd

using namespace wsvd;

extern "C" size_t wsvd_decode_multi_workspace_size(int B, int Tq, int Hq, int Hkv, int r, int L_cap) {
  if (B < 0 || Tq < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || r < 1 || L_cap < 0) return 0;
  return grouped_shape(B, Tq, Hq, Hkv, r, L_cap).total;
}

extern "C" int wsvd_decode_multi(int B, int Tq, int Hq, int Hkv, int Hd, int r, int bits, int L_cap,
                                 const int32_t* seq_lens, const void* q, int q_dtype, const uint8_t* lat_k,
                                 const uint8_t* lat_v, const void* scale_k, const void* scale_v, const void* B_k,
                                 const void* B_v, float softmax_scale, float* out, void* workspace,
                                 size_t workspace_bytes, int32_t* err, void* stream) {
  if (B < 0 || Tq < 1 || Hq < 1 || Hkv < 1 || L_cap < 0 || Hq % Hkv) return WSVD_ERR_INVALID_ARG;
  if (B == 0) return WSVD_OK;
  const int G = Hq / Hkv;
  if (G * Tq > 64) return WSVD_ERR_UNSUPPORTED;
  if (B > 65535) return WSVD_ERR_UNSUPPORTED;
  if (Hd != 32 && Hd != 64 && Hd != 128 && Hd != 256) return WSVD_ERR_UNSUPPORTED;
  if (L_cap % 8) return WSVD_ERR_UNSUPPORTED;
  if (bits != 8 && bits != 4) return WSVD_ERR_INVALID_ARG;
  if (r < 1 || (r * bits) % 8) return WSVD_ERR_INVALID_ARG;
  const int rb = r * bits / 8;
  if (rb != 16 && rb != 32 && rb != 64) return WSVD_ERR_UNSUPPORTED;
  if (q_dtype != WSVD_DTYPE_FP16 && q_dtype != WSVD_DTYPE_BF16) return WSVD_ERR_INVALID_ARG;
  if (!seq_lens || !q || !lat_k || !lat_v || !scale_k || !scale_v || !B_k || !B_v || !out || !workspace)
    return WSVD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(lat_k) || !aligned16(lat_v) || !aligned16(scale_k) || !aligned16(scale_v) ||
      !aligned16(B_k) || !aligned16(B_v) || !aligned16(out) || !aligned16(workspace))
    return WSVD_ERR_INVALID_ARG;
  const GroupedShape sh = grouped_shape(B, Tq, Hq, Hkv, r, L_cap);
  if ((size_t)Hkv * sh.nqc > 65535) return WSVD_ERR_UNSUPPORTED;
  if (workspace_bytes < sh.total) return WSVD_ERR_WORKSPACE_TOO_SMALL;
  GroupedKernels gk{};
  if (!pick_grouped(bits, rb, sh.nq, &gk)) return WSVD_ERR_UNSUPPORTED;
  const size_t smem = gk.smem;
  int sms = 148, occ = 1;
  if (device_setup(gk.decode, smem, gk.tmem_ctas, &sms, &occ) != cudaSuccess) return WSVD_ERR_CUDA;

  GroupedArgs ga{};
  ga.B = B; ga.Tq = Tq; ga.Hq = Hq; ga.Hkv = Hkv; ga.G = G; ga.Hd = Hd; ga.L_cap = L_cap;
  ga.nqc = sh.nqc;
  const int tiles_cap = std::max(1, (L_cap + kGTok - 1) / kGTok);
  const long long groups = (long long)B * Hkv * sh.nqc;
  const int nsplit = grouped_splits(groups, tiles_cap, sh.slots, sms, occ);
  ga.chunk_tiles = (tiles_cap + nsplit - 1) / nsplit;
  ga.nsplit = (tiles_cap + ga.chunk_tiles - 1) / ga.chunk_tiles;
  ga.slot_stride = sh.slots;
  ga.seq_lens = seq_lens; ga.q = q; ga.q_dtype = q_dtype;
  ga.lat_k = lat_k; ga.lat_v = lat_v;
  ga.scale_k = static_cast<const __half*>(scale_k); ga.scale_v = static_cast<const __half*>(scale_v);
  ga.Bk = static_cast<const __half*>(B_k); ga.Bv = static_cast<const __half*>(B_v);
  ga.qscale = (softmax_scale != 0.f ? softmax_scale : (float)(1.0 / sqrt((double)Hd))) * 1.4426950408889634f;
  ga.out = out;
  ga.partials = static_cast<float*>(workspace);
  ga.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + sh.partial_bytes);
  uint8_t* planes = static_cast<uint8_t*>(workspace) + sh.partial_bytes + sh.counter_bytes;
  ga.qplanes = planes;
  ga.err = err;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  {  // q' planes of every query group
    void* pargs[] = {&ga, &planes};
    const size_t psmem = qproj_smem_bytes(r, sh.nq, Hd);
    if (cudaFuncSetAttribute(gk.qproj, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem) != cudaSuccess)
      return WSVD_ERR_CUDA;
    cudaLaunchConfig_t pcfg = {};
    pcfg.gridDim = dim3((unsigned)groups);
    pcfg.blockDim = dim3(128);
    pcfg.dynamicSmemBytes = psmem;
    pcfg.stream = st;
    if (cudaLaunchKernelExC(&pcfg, gk.qproj, pargs) != cudaSuccess) return WSVD_ERR_CUDA;
  }
  // The decode grid behind it as a programmatic dependent: it starts streaming
  // tiles while the projection runs and stages the planes after griddepcontrol.wait.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  void* args[] = {&ga};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ga.nsplit, Hkv * sh.nqc, B);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, gk.decode, args) == cudaSuccess ? WSVD_OK : WSVD_ERR_CUDA;
}

extern "C" size_t wsvd_decode_gqa_workspace_size(int B, int Hq, int Hkv, int r, int L_cap) {
  return wsvd_decode_multi_workspace_size(B, 1, Hq, Hkv, r, L_cap);
}

extern "C" int wsvd_decode_gqa(int B, int Hq, int Hkv, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                               const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                               const void* scale_k, const void* scale_v, const void* B_k, const void* B_v,
                               float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                               int32_t* err, void* stream) {
  return wsvd_decode_multi(B, 1, Hq, Hkv, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v,
                           B_k, B_v, softmax_scale, out, workspace, workspace_bytes, err, stream);
}
