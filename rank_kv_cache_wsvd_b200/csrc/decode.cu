// Persistent split-L flash-decoding over a low-rank (int8 / int4) or dense
// (fp16) cache, for sm_100a.  One launch does the whole decode step.
//
// The fused decode of the WSVD summaries (Japanese §2.4, German §2.D) streams
// tiles of each head's latent cache C_Kh through on-chip memory and runs
// q.K^T, softmax and the V product without writing K or V out.  Here the K/V
// reconstruction through B_Kh / B_Vh is reassociated onto the query and the
// output:
//     q'    = B_Kh . q                               (once per (b, h))
//     s_l   = s^K_l (code^K_l . q') * softmax_scale   (r values per token)
//     o_lat = sum_l p_l s^V_l code^V_l,  out = (o_lat / sum_l p_l) . B_Vh
// so the per-token work is O(r) instead of O(r * Hd) and the only bytes read
// per token are its 2 x r codes and 2 fp16 scales.
//
// Arithmetic per token.  K side: q' is held as a 24-bit fixed-point integer
// split into three byte planes, so code . q' is three dp4a chains (exact
// integer sums) combined once in fp32; the fixed-point step is max|q'| / 2^23.
// V side: codes are turned into exact fp32 values by placing them in the
// mantissa of 2^23 (one byte-permute or bit-select per code) and accumulated
// with packed fp32x2 FMAs.
//
// Work decomposition: the (b, h, tile) space of all sequences is flattened
// (tiles of T tokens, t fastest) and split evenly over a persistent grid of C
// CTAs, so ragged lengths cost nothing extra.  A CTA that owns all tiles of a
// (b, h) finishes it alone; otherwise each CTA writes one partial (m, l,
// o[W]) into slot c + b*H + h (slots of consecutive CTAs never collide because
// tile ranges are ordered) and bumps a per-(b, h) counter; the CTA that
// arrives last merges the partials and applies B_Vh (last-arriver pattern, no
// waiting), then resets the counter to zero.
//
// Small problems (few tiles per resident CTA) use decode_cluster_kernel
// instead: one thread-block cluster per (b, h) splits the tokens and merges
// through distributed shared memory (see below).
//
// Per CTA of the persistent kernel: one producer warp issues 1-D bulk copies
// (TMA, no multicast) of
// K codes, V codes and their scales into a shared-memory ring; eight consumer
// warps each own NTOK tokens per tile (TPT adjacent lanes per token, VPT
// values per lane), keep a per-lane online softmax and reduce across lanes /
// warps only at (b, h) boundaries.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include <cooperative_groups.h>

#include "append_core.cuh"
#include "common.cuh"

namespace cg = cooperative_groups;

namespace wsvd {

template <int CODEC>
struct CodecT;
template <>
struct CodecT<kCodecI8> {
  static constexpr int kBits = 8;
  static constexpr bool kScaled = true;
};
template <>
struct CodecT<kCodecI4> {
  static constexpr int kBits = 4;
  static constexpr bool kScaled = true;
};
template <>
struct CodecT<kCodecF16> {
  static constexpr int kBits = 16;
  static constexpr bool kScaled = false;
};

constexpr int kMaxClusterSize = 8;

// Per-(b, h) operands the producer stages next to the tiles: B_Kh and q (low-rank
// path), q (dense path) or the projected q' (shared-latent path).  Two buffers
// when they are small, so the next segment's operands load under the current one.
__host__ __device__ inline size_t seg_bytes(int qmode, int W, int Hd) {
  size_t b = qmode == kQProj ? (size_t)W * Hd * 2 + (size_t)Hd * 2 : (qmode == kQDirect ? (size_t)Hd * 2 : (size_t)W * 4);
  return (b + 127) / 128 * 128;
}
__host__ __device__ inline int seg_nbuf(int qmode, int W, int Hd) { return seg_bytes(qmode, W, Hd) <= 17408 ? 2 : 1; }

// Helper-owned shared state (after the operand buffers): NQ query-state slots
// the helper fills ahead of the consumers, two result slots it drains.
template <int W, int PW, int NQ>
struct HelperArea {
  float qsv[NQ][W];           // scaled q' (fp16 codecs read it directly)
  uint32_t planes[NQ][PW];    // packed byte planes + int4 corrections
  float qstep[NQ];
  int seginfo[NQ][4];         // b, h, c_first, c_last
  float res[2][W + 2];        // merged (M, L, O[W]) of a segment, consumers -> helper
  int qi[W];                  // quantised q'
  uint64_t bars[2 * NQ + 4];  // qready[NQ], qfree[NQ], resfull[2], resfree[2]
};

// SOVR: stage count override (0: as many stages as the ring budget holds).
template <int CODEC, int VPT, int TPT, int NTOK, int SOVR = 0>
struct Cfg {
  using CT = CodecT<CODEC>;
  static constexpr int kCB = VPT * CT::kBits / 8;  // bytes per lane per token
  static constexpr int kNSeg = kCB / 16;           // 16-byte shared loads per lane per token
  static constexpr int kRB = kCB * TPT;            // bytes per token row
  static constexpr int kW = VPT * TPT;             // values per token row
  static constexpr int kTPP = kConsumerThreads / TPT;
  static constexpr int kT = kTPP * NTOK;           // tokens per tile
  static constexpr int kCodeBytes = kT * kRB;
  static constexpr int kScaleBytes = CT::kScaled ? kT * 2 : 0;
  static constexpr int kStageBytes = 2 * kCodeBytes + 2 * kScaleBytes;
  static constexpr int kStageBudget = kW <= 32 ? 73728 : 57344;  // ring bytes per CTA (two CTAs per SM)
  static constexpr int kStagesRaw = kStageBudget / kStageBytes;
  static constexpr int kStages =
      SOVR > 0 ? SOVR : (kStagesRaw < 2 ? 2 : (kStagesRaw > 8 ? 8 : kStagesRaw));
  static constexpr int kRedRaw = kConsumerWarps * TPT * (VPT + 2);
  static constexpr int kRedFloats = kRedRaw < kConsumerThreads ? kConsumerThreads : kRedRaw;
  static constexpr int kQW = VPT / 4;  // byte-plane words of q' per lane
  static constexpr int kNQ = kW <= 128 ? 4 : 2;  // helper query-state slots (segments built ahead)
  static_assert(kCB % 16 == 0, "a lane's chunk is a whole number of 16-byte loads");
  static_assert(kT % 8 == 0, "tile must hold a multiple of 8 tokens (16-byte scale copies)");
  static_assert(TPT <= 32 && (TPT & (TPT - 1)) == 0, "a token's lanes share a warp");
  // shared-memory layout (bytes)
  static constexpr size_t kOffBar = (size_t)kStages * kStageBytes;
  static constexpr size_t kOffQ = kOffBar + 2 * kStages * 8 + 6 * 8;  // + segment / auxiliary barriers
  static constexpr size_t kOffRed = kOffQ + (size_t)kW * 4;
  static constexpr size_t kOffRes = kOffRed + (size_t)kRedFloats * 4;
  static constexpr int kPlaneWords = TPT * (3 * kQW + 4);  // packed q' byte planes + corrections, per chunk
  static constexpr size_t kOffParts = kOffRes + (size_t)(kW + 2) * 4;
  static constexpr size_t kOffMisc = kOffParts + (size_t)kPlaneWords * 4;
  static constexpr size_t kOffPre = kOffMisc + 16 * 4;
  // runtime part: lens / prefix (2B + 1 ints), then the segment buffers
  __host__ __device__ static size_t seg_off(int B) { return (kOffPre + (size_t)(2 * B + 1) * 4 + 127) / 128 * 128; }
  // B_Vh of the CTA's last segment, staged for its finish (low-rank codecs, up
  // to 16 KB so that two CTAs still fit an SM; larger ones read global memory).
  __host__ __device__ static size_t bv_stage_bytes(int Hd) {
    return (CT::kScaled && (size_t)kW * Hd * 2 <= 16384) ? (size_t)kW * Hd * 2 : 0;
  }
  static size_t smem_bytes(int B, int qmode, int Hd) {
    return seg_off(B) + seg_nbuf(qmode, kW, Hd) * seg_bytes(qmode, kW, Hd) +
           (sizeof(HelperArea<kW, kPlaneWords, kNQ>) + 127) / 128 * 128 + bv_stage_bytes(Hd);
  }
  // cluster kernel: operands, the leader's partial slots, then B_Vh
  __host__ __device__ static size_t cluster_seg_off() { return (kOffPre + 127) / 128 * 128; }
  __host__ __device__ static size_t cluster_smem_bytes(int qmode, int Hd) {
    return cluster_seg_off() + seg_bytes(qmode, kW, Hd) + (size_t)kMaxClusterSize * (kW + 2) * 4 +
           (qmode == kQDirect ? 0 : (size_t)kW * Hd * 2);
  }
};

// ------------------------------------------------------------------ per-lane query state
template <int CODEC, int VPT>
struct QState;

template <int VPT>
struct QState<kCodecI8, VPT> {
  uint32_t qh[VPT / 4], qm[VPT / 4], ql[VPT / 4];  // signed high byte, unsigned middle / low bytes
  float step;
  // Lanes that read their chunk's two 16-byte halves in swapped order (see
  // load_chunk) hold their plane words in that order too.
  __device__ __forceinline__ void swap_halves(bool sw) {
    constexpr int H = VPT / 8;
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const uint32_t h0 = qh[k], m0 = qm[k], l0 = ql[k];
      qh[k] = sw ? qh[k + H] : h0;
      qh[k + H] = sw ? h0 : qh[k + H];
      qm[k] = sw ? qm[k + H] : m0;
      qm[k + H] = sw ? m0 : qm[k + H];
      ql[k] = sw ? ql[k + H] : l0;
      ql[k + H] = sw ? l0 : ql[k + H];
    }
  }
  __device__ __forceinline__ float dot(const uint4* seg) const {
    int ah[2] = {0, 0}, am[2] = {0, 0}, al[2] = {0, 0};  // two chains per plane
#pragma unroll
    for (int k = 0; k < VPT / 4; ++k) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(seg)[k];
      ah[k & 1] = dp4a_ss(w, qh[k], ah[k & 1]);
      am[k & 1] = dp4a_su(w, qm[k], am[k & 1]);
      al[k & 1] = dp4a_su(w, ql[k], al[k & 1]);
    }
    return fmaf((float)(ah[0] + ah[1]), 65536.f, fmaf((float)(am[0] + am[1]), 256.f, (float)(al[0] + al[1])));
  }
};

template <int VPT>
struct QState<kCodecI4, VPT> {
  // byte plane word 2k holds the even elements of source word k, 2k+1 the odd ones
  uint32_t qh[VPT / 4], qm[VPT / 4], ql[VPT / 4];
  int ch, cm, cl;  // 8 * sum of each plane: removes the +8 offset of the nibbles
  float step;
  __device__ __forceinline__ void swap_halves(bool) {}
  __device__ __forceinline__ float dot(const uint4* seg) const {
    int ah[2] = {-ch, 0}, am[2] = {-cm, 0}, al[2] = {-cl, 0};  // even / odd elements on separate chains
#pragma unroll
    for (int k = 0; k < VPT / 8; ++k) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(seg)[k];
      const uint32_t ev = (w & 0x0F0F0F0Fu) ^ 0x08080808u;         // c + 8 of elements 8k, 8k+2, ...
      const uint32_t od = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;  // c + 8 of elements 8k+1, 8k+3, ...
      ah[0] = dp4a_us(ev, qh[2 * k], ah[0]);
      ah[1] = dp4a_us(od, qh[2 * k + 1], ah[1]);
      am[0] = dp4a_uu(ev, qm[2 * k], am[0]);
      am[1] = dp4a_uu(od, qm[2 * k + 1], am[1]);
      al[0] = dp4a_uu(ev, ql[2 * k], al[0]);
      al[1] = dp4a_uu(od, ql[2 * k + 1], al[1]);
    }
    return fmaf((float)(ah[0] + ah[1]), 65536.f, fmaf((float)(am[0] + am[1]), 256.f, (float)(al[0] + al[1])));
  }
};

template <int VPT>
struct QState<kCodecF16, VPT> {
  float2 qv[VPT / 2];
  float step;
  __device__ __forceinline__ void swap_halves(bool sw) {
    constexpr int H = VPT / 4;
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const float2 t = qv[k];
      qv[k] = sw ? qv[k + H] : t;
      qv[k + H] = sw ? t : qv[k + H];
    }
  }
  __device__ __forceinline__ float dot(const uint4* seg) const {
    float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < VPT / 4; ++k) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(seg) + 2 * k;
      d0 = __ffma2_rn(h2_pair(w[0]), qv[2 * k], d0);
      d1 = __ffma2_rn(h2_pair(w[1]), qv[2 * k + 1], d1);
    }
    return (d0.x + d0.y) + (d1.x + d1.y);
  }
};

// acc[VPT/2] += wt * values(seg)
template <int CODEC, int VPT>
__device__ __forceinline__ void axpy(const uint4* seg, float wt, float2* acc) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(seg);
  if (CODEC == kCodecI8) {
    const float2 w2 = make_float2(wt, wt);
#pragma unroll
    for (int k = 0; k < VPT / 4; ++k) {
      const uint32_t x = w[k] ^ 0x80808080u;
      acc[2 * k] = __ffma2_rn(i8_pair(x, 0), w2, acc[2 * k]);
      acc[2 * k + 1] = __ffma2_rn(i8_pair(x, 2), w2, acc[2 * k + 1]);
    }
  } else if (CODEC == kCodecI4) {
    // Nibble k of a 16-bit half lands at bits 4k of the mantissa of 2^23, i.e.
    // value 2^23 + 16^k (c + 8); the weight carries the matching 16^-k.
    const float2 wa = make_float2(wt, wt * 0.0625f), wb = make_float2(wt * 0.00390625f, wt * 0.000244140625f);
    const float2 oa = make_float2(-8388616.f, -8388736.f), ob = make_float2(-8390656.f, -8421376.f);
#pragma unroll
    for (int k = 0; k < VPT / 8; ++k) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const uint32_t x = hlf ? (w[k] >> 16) : w[k];
        float2 f01, f23;
        f01.x = __uint_as_float((x & 0x000Fu) ^ 0x4B000008u);
        f01.y = __uint_as_float((x & 0x00F0u) ^ 0x4B000080u);
        f23.x = __uint_as_float((x & 0x0F00u) ^ 0x4B000800u);
        f23.y = __uint_as_float((x & 0xF000u) ^ 0x4B008000u);
        acc[4 * k + 2 * hlf] = __ffma2_rn(__fadd2_rn(f01, oa), wa, acc[4 * k + 2 * hlf]);
        acc[4 * k + 2 * hlf + 1] = __ffma2_rn(__fadd2_rn(f23, ob), wb, acc[4 * k + 2 * hlf + 1]);
      }
    }
  } else {
    const float2 w2 = make_float2(wt, wt);
#pragma unroll
    for (int k = 0; k < VPT / 2; ++k) acc[k] = __ffma2_rn(h2_pair(w[k]), w2, acc[k]);
  }
}

// ------------------------------------------------------------------ tile bookkeeping
struct TileWalk {
  const int* pre;  // pre[b] = tiles of sequences < b (per head), pre[B] = total
  int B, H;
  __device__ __forceinline__ int tiles(int b) const { return pre[b + 1] - pre[b]; }
  // (b, h, t) of flat tile g: the largest b with H * pre[b] <= g has tiles.
  __device__ __forceinline__ void locate(long long g, int& b, int& h, int& t) const {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)H * pre[mid] <= g) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    const long long rem = g - (long long)H * pre[b];
    const int tb = tiles(b);
    h = (int)(rem / tb);
    t = (int)(rem % tb);
  }
  __device__ __forceinline__ void advance(int& b, int& h, int& t) const {
    if (++t == tiles(b)) {
      t = 0;
      if (++h == H) {
        h = 0;
        do {
          ++b;
        } while (b < B && tiles(b) == 0);
      }
    }
  }
};

__device__ __forceinline__ int clamp_len(int n, int L_cap) { return (n < 0 || n > L_cap) ? 0 : n; }

// CTA that owns flat tile g when G tiles are split evenly over C CTAs.
__device__ __forceinline__ int cta_of(long long g, long long G, int C) {
  return (int)(((g + 1) * C + G - 1) / G - 1);
}

// A lane's chunk of a token row from shared memory.  With two 16-byte halves,
// lanes 4-7 of each 8-lane phase take the halves in the other order, so the
// phase touches 32 distinct banks.
__device__ __forceinline__ bool swapped_lane(int lane) { return (lane >> 2) & 1; }

template <int NSEG>
__device__ __forceinline__ void load_chunk(uint4* seg, const uint8_t* p, int lane) {
  const uint32_t a = smem_u32(p);
  if constexpr (NSEG == 2) {
    // Lanes 4-7 of every eight read the second half first (rows of 32 bytes
    // would otherwise put two lanes of a quarter-warp on the same banks).
    // The halves stay in that order: those lanes keep their query state and
    // accumulators permuted to match (swap_halves, reduce_to_res).
    const uint32_t off = swapped_lane(lane) ? 16u : 0u;
    seg[0] = lds128(a + off);
    seg[1] = lds128(a + (off ^ 16u));
  } else {
#pragma unroll
    for (int j = 0; j < NSEG; ++j) seg[j] = lds128(a + 16u * j);
  }
}

// Consumer-group barrier (the producer warp never joins).
__device__ __forceinline__ void csync() { named_barrier_sync(1, kConsumerThreads); }

// ------------------------------------------------------------------ consumer building blocks
// Builds this lane's query state from the staged per-(b, h) operands (see
// seg_bytes).  Low-rank path: q' = B_Kh . q in shared memory (eight lanes per
// row, scaled by softmax_scale * log2 e), then the lane's 24-bit fixed-point
// byte planes (step = max|q'| / 2^23).  fp16 paths: q or the projected q'.
// Contains consumer-group barriers.
// q'[j] = (B_Kh . q)[j] * qscale for rows j = j0, j0 + jstep, ...: eight lanes per
// row (part = lane & 7) sum columns part, part + 8, ... from a row-dependent
// rotation (distinct banks across the warp's rows), then a fixed shuffle tree.
// Every builder uses this routine, so q' is bit-identical whoever builds it.
// Returns this lane's max |q'| over its rows.
__device__ __forceinline__ float qprime_rows(const uint8_t* sbuf, float* qs, const DecodeArgs& a, int h, int W,
                                            int j0, int jstep, int part) {
  const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(sbuf + (size_t)W * a.Hd * (a.w8 ? 1 : 2));
  // int8 B_K: its column scales (staged after q) are folded into q
  const float* colscale = a.w8 ? reinterpret_cast<const float*>(qsrc + a.Hd) : nullptr;
  const int cols = a.Hd >> 3;  // 4, 8, 16 or 32: a power of two, a multiple of 4
  const int cmask = cols - 1;
  float amax = 0.f;
  auto qval = [&](int col) {
    const uint16_t qu = qsrc[col];
    return (a.q_dtype == WSVD_DTYPE_BF16) ? __uint_as_float((uint32_t)qu << 16) : __half2float(__ushort_as_half(qu));
  };
  for (int j = j0; j < W; j += jstep) {
    float d = 0.f;
    // columns ((k + j) mod cols) * 8 + part for k = 0, 1, ...: four loads ahead of four fmas
    if (colscale) {  // int8 B_K
      const int8_t* row = reinterpret_cast<const int8_t*>(sbuf) + (size_t)j * a.Hd;
      for (int k = 0; k < cols; k += 4) {
        float bv[4], qv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = ((k + i + j) & cmask) * 8 + part;
          bv[i] = (float)row[col];
          qv[i] = qval(col) * colscale[col];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) d = fmaf(bv[i], qv[i], d);
      }
    } else {
      const __half* row = reinterpret_cast<const __half*>(sbuf) + (size_t)j * a.Hd;
      for (int k = 0; k < cols; k += 4) {
        float bv[4], qv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = ((k + i + j) & cmask) * 8 + part;
          bv[i] = __half2float(row[col]);
          qv[i] = qval(col);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) d = fmaf(bv[i], qv[i], d);
      }
    }
    d += __shfl_xor_sync(0xffffffffu, d, 1);
    d += __shfl_xor_sync(0xffffffffu, d, 2);
    d += __shfl_xor_sync(0xffffffffu, d, 4);
    d *= a.qscale;
    amax = fmaxf(amax, fabsf(d));
    if (part == 0) qs[j] = d;
  }
  return amax;
}

template <int CODEC, int VPT, int W, int QMODE>
__device__ __forceinline__ void build_query(QState<CODEC, VPT>& qst, const uint8_t* sbuf, float* qs, float* misc,
                                            uint32_t* planes, const DecodeArgs& a, int tid, int sub) {
  using CT = CodecT<CODEC>;
  constexpr int QW = VPT / 4;
  const int warp = tid >> 5, lane = tid & 31;
  float amax = 0.f;
  if (QMODE == kQProj) {
    amax = qprime_rows(sbuf, qs, a, blockIdx.y, W, tid >> 3, kConsumerThreads / 8, tid & 7);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  } else if (QMODE == kQDirect) {
    const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(sbuf);
    for (int j = tid; j < W; j += kConsumerThreads)
      qs[j] = (a.q_dtype == WSVD_DTYPE_BF16 ? __uint_as_float((uint32_t)qsrc[j] << 16)
                                            : __half2float(__ushort_as_half(qsrc[j]))) * a.qscale;
  } else {
    const float* qg = reinterpret_cast<const float*>(sbuf);
    for (int j = tid; j < W; j += kConsumerThreads) qs[j] = qg[j] * a.qscale;
  }
  if (CT::kScaled && lane == 0) misc[warp] = amax;
  csync();
  if constexpr (CT::kScaled) {
    constexpr int TPT = W / VPT;
    float M = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, misc[w]);
    const float inv = M > 0.f ? 8388607.f / M : 0.f;
    qst.step = M > 0.f ? M / 8388607.f : 0.f;
    auto qint = [&](int e) {
      const int x = __float2int_rn(qs[e] * inv);
      return max(-8388607, min(8388607, x));
    };
    // Pack each (chunk, plane word) once: planes[(s*3 + plane)*QW + k].
    for (int idx = tid; idx < TPT * QW; idx += kConsumerThreads) {
      const int s2 = idx / QW, k = idx % QW;
      uint32_t h4 = 0, m4 = 0, l4 = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // int8: element 4k+i; int4: even/odd elements of source word k/2
        const int e = s2 * VPT + (CODEC == kCodecI8 ? 4 * k + i : 8 * (k >> 1) + 2 * i + (k & 1));
        const int x = qint(e);
        h4 |= ((uint32_t)(x >> 16) & 0xFFu) << (8 * i);
        m4 |= ((uint32_t)(x >> 8) & 0xFFu) << (8 * i);
        l4 |= ((uint32_t)x & 0xFFu) << (8 * i);
      }
      planes[(s2 * 3 + 0) * QW + k] = h4;
      planes[(s2 * 3 + 1) * QW + k] = m4;
      planes[(s2 * 3 + 2) * QW + k] = l4;
    }
    if (CODEC == kCodecI4) {
      // 8 * sum of each plane over the chunk: removes the +8 offset of the nibbles
      for (int s2 = tid; s2 < TPT; s2 += kConsumerThreads) {
        int sh = 0, sm = 0, sl = 0;
        for (int v = 0; v < VPT; ++v) {
          const int x = qint(s2 * VPT + v);
          sh += x >> 16;
          sm += (x >> 8) & 0xFF;
          sl += x & 0xFF;
        }
        planes[TPT * 3 * QW + s2 * 3 + 0] = (uint32_t)(8 * sh);
        planes[TPT * 3 * QW + s2 * 3 + 1] = (uint32_t)(8 * sm);
        planes[TPT * 3 * QW + s2 * 3 + 2] = (uint32_t)(8 * sl);
      }
    }
    csync();
#pragma unroll
    for (int k = 0; k < QW; ++k) {
      qst.qh[k] = planes[(sub * 3 + 0) * QW + k];
      qst.qm[k] = planes[(sub * 3 + 1) * QW + k];
      qst.ql[k] = planes[(sub * 3 + 2) * QW + k];
    }
    if constexpr (CODEC == kCodecI4) {
      qst.ch = (int)planes[TPT * 3 * QW + sub * 3 + 0];
      qst.cm = (int)planes[TPT * 3 * QW + sub * 3 + 1];
      qst.cl = (int)planes[TPT * 3 * QW + sub * 3 + 2];
    }
  } else {
#pragma unroll
    for (int p = 0; p < VPT / 2; ++p) qst.qv[p] = make_float2(qs[sub * VPT + 2 * p], qs[sub * VPT + 2 * p + 1]);
    qst.step = 1.f;
  }
  if constexpr (Cfg<CODEC, VPT, W / VPT, 1>::kNSeg == 2) qst.swap_halves(swapped_lane(tid & 31));
}

// One staged tile: scores, lazy-rescaled online softmax and the latent P.V
// accumulation of this lane's NTOK tokens.  Tokens n0 <= tok < n are valid
// (n0 > 0: the rest of a tile whose first rows were processed before).
template <int CODEC, int VPT, int TPT, int NTOK>
__device__ __forceinline__ void process_tile(const uint8_t* st, int n, const QState<CODEC, VPT>& qst, float& m,
                                             float& l, float2* acc, int tid, int n0 = 0) {
  using C = Cfg<CODEC, VPT, TPT, NTOK>;
  using CT = typename C::CT;
  constexpr int T = C::kT, RB = C::kRB, CB = C::kCB, NSEG = C::kNSeg, TPP = C::kTPP, NP = VPT / 2;
  const int g_tok = tid / TPT, sub = tid % TPT, lane = tid & 31;
  const __half* sck = reinterpret_cast<const __half*>(st + 2 * C::kCodeBytes);
  float sc[NTOK];
  float tmax = kNegInf;
#pragma unroll
  for (int k = 0; k < NTOK; ++k) {
    const int tok = k * TPP + g_tok;
    uint4 seg[NSEG];
    load_chunk<NSEG>(seg, st + (size_t)tok * RB + sub * CB, lane);
    float d = qst.dot(seg);
#pragma unroll
    for (int o = 1; o < TPT; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    const bool valid = tok >= n0 && tok < n;
    const float skk = (CT::kScaled && valid) ? lds_half_as_float(smem_u32(sck + tok)) * qst.step : qst.step;
    sc[k] = valid ? d * skk : kNegInf;
    tmax = fmaxf(tmax, sc[k]);
  }
  if (tmax > m + 8.f) {  // lazy rescale: the reference moves only when a score beats it by 2^8
    const float fr = ex2(m - tmax);
    l *= fr;
#pragma unroll
    for (int p = 0; p < NP; ++p) acc[p] = __fmul2_rn(acc[p], make_float2(fr, fr));
    m = tmax;
  }
#pragma unroll
  for (int k = 0; k < NTOK; ++k) {
    const int tok = k * TPP + g_tok;
    if (tok >= n0 && tok < n) {
      const float p = ex2(sc[k] - m);
      l += p;
      const float wv = CT::kScaled ? p * lds_half_as_float(smem_u32(sck + T + tok)) : p;
      uint4 seg[NSEG];
      load_chunk<NSEG>(seg, st + C::kCodeBytes + (size_t)tok * RB + sub * CB, lane);
      axpy<CODEC, VPT>(seg, wv, acc);
    }
  }
}

// Butterfly reduce-scatter across the lanes that share a chunk (lane offsets
// O, O/2, ..., TPT): each round a lane keeps half of its values and adds the
// partner's matching half, so the values to move halve every round.
template <int CUR, int O, int TPT>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
  if constexpr (O >= TPT) {
    if constexpr (CUR >= 2) {
      constexpr int HALF = CUR / 2;
      const bool up = lane & O;
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        const float send = up ? v[j] : v[j + HALF];
        const float keep = up ? v[j + HALF] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      reduce_scatter<HALF, O / 2, TPT>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      reduce_scatter<1, O / 2, TPT>(v, lane);
    }
  }
}

// First element index held by a lane after reduce_scatter (values j = 0.. are consecutive).
template <int CUR, int O, int TPT>
__device__ __forceinline__ int scatter_base(int lane) {
  if constexpr (O >= TPT && CUR >= 2) {
    return ((lane & O) ? CUR / 2 : 0) + scatter_base<CUR / 2, O / 2, TPT>(lane);
  } else {
    return 0;
  }
}

// Merges every consumer lane's (m, l, acc) into res[] = (M, L, O[W]): a common
// maximum per chunk, a butterfly reduce-scatter inside each warp, then the
// eight warps through red[] (8*W floats of warp partials, then (M, l) pairs).
template <int VPT, int TPT, int W, int NSEG>
__device__ __forceinline__ void reduce_to_res(float m, float l, float2* acc, float* red, float* res, int tid) {
  constexpr int NP = VPT / 2;
  constexpr int FINAL = (VPT * TPT >= 32) ? VPT * TPT / 32 : 1;
  const int warp = tid >> 5, lane = tid & 31, sub = tid % TPT;
  float M = m;
#pragma unroll
  for (int o = TPT; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float f = (m == kNegInf) ? 0.f : ex2(m - M);
  l *= f;
#pragma unroll
  for (int o = TPT; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  float v[VPT];
  const bool sw = NSEG == 2 && swapped_lane(lane);  // accumulators of a swapped lane hold the halves permuted
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const float2 x = (NSEG == 2 && sw) ? acc[p ^ (NP / 2)] : acc[p];
    v[2 * p] = x.x * f;
    v[2 * p + 1] = x.y * f;
  }
  reduce_scatter<VPT, 16, TPT>(v, lane);
  const int base = sub * VPT + scatter_base<VPT, 16, TPT>(lane);
  float* wp = red + (size_t)warp * W;
#pragma unroll
  for (int j = 0; j < FINAL; ++j) wp[base + j] = v[j];
  float* ml = red + (size_t)kConsumerWarps * W;
  if (lane == 0) {
    ml[2 * warp] = M;
    ml[2 * warp + 1] = l;
  }
  csync();
  float Mg = kNegInf;
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) Mg = fmaxf(Mg, ml[2 * w]);
  float fw[kConsumerWarps];
#pragma unroll
  for (int w = 0; w < kConsumerWarps; ++w) fw[w] = (ml[2 * w] == kNegInf) ? 0.f : ex2(ml[2 * w] - Mg);
  for (int e = tid; e < W; e += kConsumerThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) s = fmaf(fw[w], red[(size_t)w * W + e], s);
    res[2 + e] = s;
  }
  if (tid == 0) {
    float ls = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) ls = fmaf(fw[w], ml[2 * w + 1], ls);
    res[0] = Mg;
    res[1] = ls;
  }
  csync();
}

// Merges rows p < np of a partial array part[p][W + 2] = (m, l, o[W]) into
// res[]: M = max_p m_p, then for every element (l, o[0..W)) the sum over p in
// ascending order of 2^(m_p - M) * value.  Each element is computed by one
// thread with the same operation order whatever the thread count, so a
// warp and a thread block give identical bits.  ldcg selects L2-coherent
// loads (rows written by other CTAs).
template <int W, bool GLOBAL>
__device__ __forceinline__ float merge_elem(const float* part, int np, float M, int e) {
  float s2 = 0.f;
  auto term = [&](int p) {
    const float mp = GLOBAL ? __ldcg(part + (size_t)p * (W + 2)) : part[(size_t)p * (W + 2)];
    if (mp != kNegInf) {
      const float v = GLOBAL ? __ldcg(part + (size_t)p * (W + 2) + 1 + e) : part[(size_t)p * (W + 2) + 1 + e];
      s2 = fmaf(ex2(mp - M), v, s2);
    }
  };
  if constexpr (GLOBAL) {
    for (int p = 0; p < np; ++p) term(p);
  } else {  // a cluster's ranks: at most kMaxClusterSize rows, unrolled (same order)
#pragma unroll
    for (int p = 0; p < kMaxClusterSize; ++p)
      if (p < np) term(p);
  }
  return s2;
}
template <int W, bool GLOBAL>
__device__ __forceinline__ float merge_max(const float* part, int np) {
  float M = kNegInf;
  if constexpr (GLOBAL) {
    for (int p = 0; p < np; ++p) M = fmaxf(M, __ldcg(part + (size_t)p * (W + 2)));
  } else {
#pragma unroll
    for (int p = 0; p < kMaxClusterSize; ++p)
      if (p < np) M = fmaxf(M, part[(size_t)p * (W + 2)]);
  }
  return M;
}
// Thread-block version (consumer threads).
template <int W, bool GLOBAL>
__device__ __forceinline__ void merge_rows(const float* part, int np, float* res, int tid) {
  const float M = merge_max<W, GLOBAL>(part, np);
  for (int e = tid; e < W + 1; e += kConsumerThreads) res[1 + e] = merge_elem<W, GLOBAL>(part, np, M, e);
  if (tid == 0) res[0] = M;
  csync();
}

// Up-projection operand: B_Vh (fp16, or int8 with per-column scales sv).
struct BvRef {
  const void* p;   // [W][Hd], or null on the dense path
  int w8;
  const float* sv;  // w8: [Hd]
};

// One output column: (sum over e ascending of O[e] * Bv[e][d]) (* sv[d] for
// int8 B_V) / L; dense path (no B_V): O[d] / L.  L = 0 (no tokens) gives zero.
template <int W>
__device__ __forceinline__ float out_col(const float* res, const BvRef& bv, int Hd, int d) {
  const float inv = res[1] > 0.f ? 1.f / res[1] : 0.f;
  if (bv.p == nullptr) return res[2 + d] * inv;
  float s = 0.f;
  if (bv.w8) {
    const int8_t* B8 = static_cast<const int8_t*>(bv.p);
    for (int e = 0; e < W; ++e) s = fmaf(res[2 + e], (float)B8[(size_t)e * Hd + d], s);
    s *= bv.sv[d];
  } else {
    const __half* Bh = static_cast<const __half*>(bv.p);
    for (int e = 0; e < W; ++e) s = fmaf(res[2 + e], __half2float(Bh[(size_t)e * Hd + d]), s);
  }
  return s * inv;
}

// out[b, h, :] from the merged res[] (consumer threads; see out_col).
template <int W>
__device__ __forceinline__ void finalize_out(const float* res, const BvRef& bv, float* outp, int Hd, float* red,
                                             int tid) {
  for (int d = tid; d < Hd; d += kConsumerThreads) outp[d] = out_col<W>(res, bv, Hd, d);
  csync();
}

// Producer: stage the per-(b, h) operands into a segment buffer.
template <int W, int QMODE>
__device__ __forceinline__ void issue_operands(uint8_t* dst, uint64_t* bar, const DecodeArgs& a, int b, int h,
                                               uint64_t keep) {
  const size_t bh = (size_t)b * a.H + h;
  if (QMODE == kQProj) {
    // B_Kh, q and (int8 B_K) its column scales; the segment buffer holds
    // W * Hd * 2 + Hd * 2 bytes, enough for the scales when B_K is int8.
    const uint32_t bb = (uint32_t)W * a.Hd * (a.w8 ? 1 : 2), qb = (uint32_t)a.Hd * 2, sb = a.w8 ? (uint32_t)a.Hd * 4 : 0u;
    mbar_arrive_expect_tx(bar, bb + qb + sb);
    bulk_g2s(dst, static_cast<const uint8_t*>(a.Bk) + (size_t)h * bb, bb, bar, keep);
    bulk_g2s(dst + bb, static_cast<const uint16_t*>(a.q) + bh * a.Hd, qb, bar, keep);
    if (a.w8) bulk_g2s(dst + bb + qb, a.sBk + (size_t)h * a.Hd, sb, bar, keep);
  } else if (QMODE == kQDirect) {
    mbar_arrive_expect_tx(bar, (uint32_t)a.Hd * 2);
    bulk_g2s(dst, static_cast<const uint16_t*>(a.q) + bh * a.Hd, (uint32_t)a.Hd * 2, bar, keep);
  } else {
    mbar_arrive_expect_tx(bar, (uint32_t)W * 4);
    bulk_g2s(dst, a.qglobal + bh * W, (uint32_t)W * 4, bar, keep);
  }
}

// Producer: stage tile t (n valid tokens) of (b, h) into ring stage st.
template <int CODEC, int VPT, int TPT, int NTOK>
__device__ __forceinline__ void issue_tile(uint8_t* st, uint64_t* bar, const DecodeArgs& a, int b, int h, int t,
                                           int n, uint64_t pol) {
  using C = Cfg<CODEC, VPT, TPT, NTOK>;
  using CT = typename C::CT;
  const size_t head_row = ((size_t)b * a.H + h) * a.L_cap + (size_t)t * C::kT;
  const size_t row0 = a.heads_share ? (size_t)b * a.L_cap + (size_t)t * C::kT : head_row;
  const uint32_t cb = (uint32_t)n * C::kRB;
  const uint32_t sb = CT::kScaled ? (uint32_t)((n + 7) & ~7) * 2u : 0u;
  mbar_arrive_expect_tx(bar, 2 * cb + 2 * sb);
  bulk_g2s(st, a.lat_k + row0 * C::kRB, cb, bar, pol);
  bulk_g2s(st + C::kCodeBytes, a.lat_v + row0 * C::kRB, cb, bar, pol);
  if (CT::kScaled) {
    bulk_g2s(st + 2 * C::kCodeBytes, a.scale_k + head_row, sb, bar, pol);
    bulk_g2s(st + 2 * C::kCodeBytes + C::kScaleBytes, a.scale_v + head_row, sb, bar, pol);
  }
}

// ------------------------------------------------------------------ persistent kernel
// Warp roles: warps 0-7 consume tiles, warp 8 is the producer (TMA), warp 9 the
// helper.  The helper builds each (b, h)'s query state (q' and its byte planes)
// one segment ahead of the consumers and finishes each segment after them
// (partial write, completion counter, last-arriver merge, B_Vh up-projection),
// so the consumers only stream tiles and reduce their own registers.

// Warp-level q' = B_Kh . q from the staged operands: lane j-rotation keeps the
// row reads on distinct banks.  Returns max|q'| (scaled by softmax_scale * log2 e).
template <int W, int QMODE>
__device__ __forceinline__ float helper_qprime(const uint8_t* sbuf, float* qsv, const DecodeArgs& a, size_t bh,
                                               int lane) {
  float amax = 0.f;
  if (QMODE == kQProj) {
    amax = qprime_rows(sbuf, qsv, a, (int)(bh % a.H), W, lane >> 3, 4, lane & 7);
  } else if (QMODE == kQDirect) {
    const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(sbuf);
    for (int j = lane; j < W; j += 32) {
      qsv[j] = (a.q_dtype == WSVD_DTYPE_BF16 ? __uint_as_float((uint32_t)qsrc[j] << 16)
                                             : __half2float(__ushort_as_half(qsrc[j]))) * a.qscale;
      amax = fmaxf(amax, fabsf(qsv[j]));
    }
  } else {  // q' projected beforehand into global memory (L2-coherent loads)
    const float* qg = a.qglobal + bh * W;
    for (int j = lane; j < W; j += 32) {
      qsv[j] = __ldcg(qg + j) * a.qscale;
      amax = fmaxf(amax, fabsf(qsv[j]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  return amax;
}

// Warp-level packing of the 24-bit fixed-point q' into byte planes (see QState).
template <int CODEC, int VPT, int W>
__device__ __forceinline__ void helper_planes(const float* qsv, int* qi, uint32_t* planes, float* qstep, float amax,
                                              int lane) {
  constexpr int TPT = W / VPT, QW = VPT / 4;
  const float inv = amax > 0.f ? 8388607.f / amax : 0.f;
  *qstep = amax > 0.f ? amax / 8388607.f : 0.f;
  for (int j = lane; j < W; j += 32) qi[j] = max(-8388607, min(8388607, __float2int_rn(qsv[j] * inv)));
  __syncwarp();
  for (int idx = lane; idx < TPT * QW; idx += 32) {
    const int s2 = idx / QW, k = idx % QW;
    uint32_t h4 = 0, m4 = 0, l4 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = s2 * VPT + (CODEC == kCodecI8 ? 4 * k + i : 8 * (k >> 1) + 2 * i + (k & 1));
      const int x = qi[e];
      h4 |= ((uint32_t)(x >> 16) & 0xFFu) << (8 * i);
      m4 |= ((uint32_t)(x >> 8) & 0xFFu) << (8 * i);
      l4 |= ((uint32_t)x & 0xFFu) << (8 * i);
    }
    planes[(s2 * 3 + 0) * QW + k] = h4;
    planes[(s2 * 3 + 1) * QW + k] = m4;
    planes[(s2 * 3 + 2) * QW + k] = l4;
  }
  if (CODEC == kCodecI4) {
    for (int s2 = 0; s2 < TPT; ++s2) {
      int sh = 0, sm = 0, sl = 0;
      for (int v = lane; v < VPT; v += 32) {
        const int x = qi[s2 * VPT + v];
        sh += x >> 16;
        sm += (x >> 8) & 0xFF;
        sl += x & 0xFF;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sh += __shfl_xor_sync(0xffffffffu, sh, o);
        sm += __shfl_xor_sync(0xffffffffu, sm, o);
        sl += __shfl_xor_sync(0xffffffffu, sl, o);
      }
      if (lane == 0) {
        planes[TPT * 3 * QW + s2 * 3 + 0] = (uint32_t)(8 * sh);
        planes[TPT * 3 * QW + s2 * 3 + 1] = (uint32_t)(8 * sm);
        planes[TPT * 3 * QW + s2 * 3 + 2] = (uint32_t)(8 * sl);
      }
    }
  }
  __syncwarp();
}

// Warp-level out[b, h, :] (same per-column arithmetic as finalize_out).
template <int W>
__device__ __forceinline__ void helper_finalize(const float* res, const BvRef& bv, float* outp, int Hd, int lane) {
  for (int d = lane; d < Hd; d += 32) outp[d] = out_col<W>(res, bv, Hd, d);
}

template <int CODEC, int VPT, int TPT, int NTOK, int QMODE>
__global__ void __launch_bounds__(kPersistThreads, 2) decode_kernel(const DecodeArgs a) {
  using C = Cfg<CODEC, VPT, TPT, NTOK>;
  using CT = typename C::CT;
  using HA = HelperArea<C::kW, C::kPlaneWords, C::kNQ>;
  constexpr int T = C::kT, W = C::kW, S = C::kStages, NP = VPT / 2, QW = VPT / 4, NQ = C::kNQ;
  constexpr int kProducerWarp = kConsumerWarps, kHelperWarp = kConsumerWarps + 1;
  // How far the helper may build ahead of the oldest unfinished segment.  With
  // q' in global memory nothing else gates a build; with operands staged by the
  // producer (dense path) it stays one ahead, the producer being at most a
  // ring's length ahead of the consumers.
  constexpr int kAhead = QMODE == kQGlobal ? NQ : 2;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + S;
  uint64_t* segfull = empty + S;  // [2]
  uint64_t* segempty = segfull + 2;
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  int* pre = reinterpret_cast<int*>(smem + C::kOffPre);
  int* lens = pre + a.B + 1;
  uint8_t* segbuf = smem + C::seg_off(a.B);
  const int NBUF = seg_nbuf(QMODE, W, a.Hd);
  const uint32_t SEGB = (uint32_t)seg_bytes(QMODE, W, a.Hd);
  HA* ha = reinterpret_cast<HA*>(segbuf + (size_t)NBUF * SEGB);
  __half* bv_last = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(ha) + (sizeof(HA) + 127) / 128 * 128);
  uint64_t* bvbar = segempty + 2;  // B_Vh of the last segment staged
  uint64_t* qready = ha->bars;
  uint64_t* qfree = ha->bars + NQ;
  uint64_t* resfull = ha->bars + 2 * NQ;
  uint64_t* resfree = ha->bars + 2 * NQ + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  // Programmatic dependent launch: behind the append (dep 2) the split plan
  // reads seq_lens, so nothing here may run before that grid has completed;
  // behind the q' projection alone (dep 1) only the helper waits, before it
  // reads q'.
  if (a.dep == 2) griddep_wait();

  // Valid lengths, tiles per sequence (per head) and their exclusive prefix.
  if (warp == 0) {
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) {
      const int raw = a.seq_lens[b];
      if ((raw < 0 || raw > a.L_cap) && c == 0) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
      const int n = clamp_len(raw, a.L_cap);
      lens[b] = n;
      sum += (n + T - 1) / T;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int b = b0; b < b1; ++b) {
      pre[b] = run;
      run += (lens[b] + T - 1) / T;
    }
    if (lane == 31) pre[a.B] = incl;
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], kConsumerWarps);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(&segfull[s], 1);
        mbar_init(&segempty[s], 1);
        mbar_init(&resfull[s], 1);
        mbar_init(&resfree[s], 1);
      }
      mbar_init(bvbar, 1);
      for (int s = 0; s < NQ; ++s) {
        mbar_init(&qready[s], 1);
        mbar_init(&qfree[s], kConsumerWarps);
      }
      fence_mbar_init();
    }
  }
  __syncthreads();

  // Sequences with no tokens get a zero output (spread over the CTAs).
  for (int b = c; b < a.B; b += a.ctas) {
    if (lens[b] == 0)
      for (int i = tid; i < a.H * a.Hd; i += blockDim.x) a.out[(size_t)b * a.H * a.Hd + i] = 0.f;
  }

  const TileWalk walk{pre, a.B, a.H};
  const long long G = (long long)a.H * pre[a.B];
  // At most one CTA per tile, so every working CTA owns at least one tile and
  // the CTAs that share a (b, h) are consecutive without gaps.
  const int CW = (int)(G < a.ctas ? G : a.ctas);
  if (c >= CW) {  // uniform across the CTA; nothing was issued
    if (a.dep == 1) griddep_wait();  // the grid never completes before the q' grid it was launched behind
    return;
  }
  const long long g_begin = G * c / CW, g_end = G * (c + 1) / CW;

  // ---------------------------------------------------------------- producer warp
  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy(), keep = l2_evict_last_policy();
      int b, h, t;
      walk.locate(g_begin, b, h, t);
      long long issued = 0;
      int nseg = 0, pb = -1, ph = -1;
      bool ok = true;
      for (long long g = g_begin; g < g_end && ok; ++g, ++issued) {
        if (QMODE != kQGlobal && (b != pb || h != ph)) {  // operands of the next (b, h)
          const int sb = nseg % NBUF;
          if (nseg >= NBUF && !mbar_wait_bounded(&segempty[sb], (uint32_t)(((nseg / NBUF) - 1) & 1))) {
            set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
            ok = false;
            break;
          }
          issue_operands<W, QMODE>(segbuf + (size_t)sb * SEGB, &segfull[sb], a, b, h, keep);
          ++nseg;
          pb = b;
          ph = h;
        }
        const int s = (int)(issued % S);
        if (issued >= S && !mbar_wait_bounded(&empty[s], (uint32_t)(((issued / S) - 1) & 1))) {
          set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
          ok = false;
          break;
        }
        issue_tile<CODEC, VPT, TPT, NTOK>(stages + (size_t)s * C::kStageBytes, &full[s], a, b, h, t,
                                          min(T, lens[b] - t * T), pol);
        walk.advance(b, h, t);
      }
      // B_Vh of the CTA's last segment, for the consumers' finish (issued after
      // the tiles so that it does not compete with the first ones).
      const bool stage_bv = C::bv_stage_bytes(a.Hd) > 0 && a.Bv != nullptr;
      if (stage_bv) {
        int lb, lh, lt;
        walk.locate(g_end - 1, lb, lh, lt);
        // B_Vh, and (int8 B_V, half the bytes) its column scales after it
        const uint32_t bytes = (uint32_t)W * a.Hd * (a.w8 ? 1 : 2), sbytes = a.w8 ? (uint32_t)a.Hd * 4 : 0u;
        mbar_arrive_expect_tx(bvbar, bytes + sbytes);
        for (uint32_t off = 0; off < bytes; off += 32768)
          bulk_g2s(reinterpret_cast<uint8_t*>(bv_last) + off,
                   static_cast<const uint8_t*>(a.Bv) + (size_t)lh * bytes + off, min(32768u, bytes - off), bvbar,
                   keep);
        if (a.w8)
          bulk_g2s(reinterpret_cast<uint8_t*>(bv_last) + bytes, a.sBv + (size_t)lh * a.Hd, sbytes, bvbar, keep);
      }
      // Leave no copy in flight behind: wait (bounded) for the last uses of each buffer.
      if (stage_bv && !mbar_wait_bounded(bvbar, 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      for (long long i = (issued > S ? issued - S : 0); i < issued && ok; ++i)
        if (!mbar_wait_bounded(&full[(int)(i % S)], (uint32_t)((i / S) & 1))) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      for (int k = (nseg > NBUF ? nseg - NBUF : 0); k < nseg && ok; ++k)
        if (!mbar_wait_bounded(&segfull[k % NBUF], (uint32_t)((k / NBUF) & 1))) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    }
    return;
  }

  // ---------------------------------------------------------------- helper warp
  if (warp == kHelperWarp) {
    int b = 0, h = 0, t = 0;
    walk.locate(g_begin, b, h, t);
    long long g = g_begin;
    // next (b, h) segment of this CTA's tile range, or false at the end
    auto next_segment = [&](int& sbk, int& shk) {
      if (g >= g_end) return false;
      sbk = b;
      shk = h;
      while (g < g_end && b == sbk && h == shk) {
        walk.advance(b, h, t);
        ++g;
      }
      return true;
    };
    bool timed_out = false;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (!mbar_wait_bounded(bar, parity, timed_out ? 0ull : kWaitLimitNs)) {
        if (!timed_out && lane == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
        timed_out = true;
      }
    };
    int built = 0, done = 0;
    bool more = true;
    if (QMODE == kQGlobal) griddep_wait();  // q' comes from the grid this one was launched behind
    while (true) {
      // Build ahead of the oldest unfinished segment (see kAhead).
      while (more && built < done + kAhead) {
        int sb_b, sb_h;
        if (!next_segment(sb_b, sb_h)) {
          more = false;
          break;
        }
        const int k = built, sq = k % NQ;
        const int tb = walk.tiles(sb_b);
        const long long gf = (long long)a.H * pre[sb_b] + (long long)sb_h * tb;
        const int cf = cta_of(gf, G, CW), cl = cta_of(gf + tb - 1, G, CW);
        if (lane == 0) {
          ha->seginfo[sq][0] = sb_b;
          ha->seginfo[sq][1] = sb_h;
          ha->seginfo[sq][2] = cf;
          ha->seginfo[sq][3] = cl;
        }
        if (a.Bv != nullptr && c == cl) {  // the likely finisher warms B_Vh in L2
          const int bytes = W * a.Hd * (a.w8 ? 1 : 2);
          const char* bv = static_cast<const char*>(a.Bv) + (size_t)sb_h * bytes;
          for (int o = lane * 128; o < bytes; o += 32 * 128) prefetch_l2(bv + o);
        }
        if (QMODE != kQGlobal) wait(&segfull[k % NBUF], (uint32_t)((k / NBUF) & 1));
        if (k >= NQ) wait(&qfree[sq], (uint32_t)(((k / NQ) - 1) & 1));
        const float amax = helper_qprime<W, QMODE>(segbuf + (size_t)(k % NBUF) * SEGB, ha->qsv[sq], a,
                                                   (size_t)sb_b * a.H + sb_h, lane);
        __syncwarp();
        if (QMODE != kQGlobal && lane == 0) mbar_arrive(&segempty[k % NBUF]);  // staged operands consumed
        if constexpr (CT::kScaled) {
          helper_planes<CODEC, VPT, W>(ha->qsv[sq], ha->qi, ha->planes[sq], &ha->qstep[sq], amax, lane);
        } else {
          if (lane == 0) ha->qstep[sq] = 1.f;
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(&qready[sq]);
        ++built;
      }
      // The consumers finish the CTA's last segment themselves.
      if (done == built || (!more && done == built - 1)) break;
      // Finish segment `done` once the consumers have reduced it.
      const int k = done, sr = k & 1, si = k % NQ;
      wait(&resfull[sr], (uint32_t)((k / 2) & 1));
      const float* res = ha->res[sr];
      const int sb_b = ha->seginfo[si][0], sb_h = ha->seginfo[si][1];
      const int cf = ha->seginfo[si][2], cl = ha->seginfo[si][3];
      float* outp = a.out + ((size_t)sb_b * a.H + sb_h) * a.Hd;
      const BvRef Bvh{a.Bv ? static_cast<const uint8_t*>(a.Bv) + (size_t)sb_h * W * a.Hd * (a.w8 ? 1 : 2) : nullptr,
                      a.w8, a.w8 ? a.sBv + (size_t)sb_h * a.Hd : nullptr};
      if (cf == cl) {
        helper_finalize<W>(res, Bvh, outp, a.Hd, lane);
      } else {
        const int bh = sb_b * a.H + sb_h;
        float* dst = a.partials + ((size_t)c + bh) * (W + 2);
        for (int e = lane; e < W + 2; e += 32) dst[e] = res[e];
        __threadfence();  // publish before the counter bump
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&a.counters[bh], 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == cl - cf) {  // last arriver: merge every partial of (b, h) in CTA order
          __threadfence();
          const int np = cl - cf + 1;
          const float* part = a.partials + ((size_t)cf + bh) * (W + 2);
          const float M = merge_max<W, true>(part, np);
          float* mres = ha->res[sr];  // reuse the segment's slot for the merged result
          for (int e = lane; e < W + 1; e += 32) mres[1 + e] = merge_elem<W, true>(part, np, M, e);
          __syncwarp();
          helper_finalize<W>(mres, Bvh, outp, a.Hd, lane);
          if (lane == 0) atomicExch(&a.counters[bh], 0);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&resfree[sr]);
      ++done;
    }
    return;
  }

  // ---------------------------------------------------------------- consumer warps
  const int sub = tid % TPT;
  QState<CODEC, VPT> qst;
  float2 acc[NP];
  float m = kNegInf, l = 0.f;
  bool timed_out = false;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (!mbar_wait_bounded(bar, parity, timed_out ? 0ull : kWaitLimitNs)) {
      if (!timed_out && lane == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      timed_out = true;
    }
  };
  int k = 0;  // segments started
  auto end_segment = [&](int j) {  // hand segment j to the helper
    const int sr = j & 1;
    if (j >= 2) wait(&resfree[sr], (uint32_t)(((j / 2) - 1) & 1));
    reduce_to_res<VPT, TPT, W, C::kNSeg>(m, l, acc, red, ha->res[sr], tid);
    if (tid == 0) mbar_arrive(&resfull[sr]);
  };
  // The CTA's last segment: every consumer thread finishes it (partial, counter,
  // last-arriver merge, up-projection); nothing runs after it.
  float* res = reinterpret_cast<float*>(smem + C::kOffRes);
  float* misc = reinterpret_cast<float*>(smem + C::kOffMisc);
  auto finish_last = [&](int b_, int h_) {
    const int tb = walk.tiles(b_);
    const long long gf = (long long)a.H * pre[b_] + (long long)h_ * tb;
    const int cf = cta_of(gf, G, CW), cl = cta_of(gf + tb - 1, G, CW);
    const int bh = b_ * a.H + h_;
    // The CTA that ends a head usually reaches it after the CTAs that start
    // it: if every other contributor has already published (the counter,
    // read with acquire, says so), this CTA is the last arriver without
    // publishing or bumping anything itself.  The read is issued before the
    // reduction so that its latency overlaps it (an early, lower count only
    // sends this CTA down the publishing path).
    const int seen = (cf != cl && tid == 0) ? ld_acquire_gpu(&a.counters[bh]) : 0;
    reduce_to_res<VPT, TPT, W, C::kNSeg>(m, l, acc, red, res, tid);
    float* outp = a.out + ((size_t)b_ * a.H + h_) * a.Hd;
    BvRef Bvh{nullptr, a.w8, a.w8 ? a.sBv + (size_t)h_ * a.Hd : nullptr};
    if (a.Bv != nullptr) {
      if (C::bv_stage_bytes(a.Hd) > 0) {  // staged by the producer (with the int8 scales after it)
        wait(bvbar, 0);
        Bvh.p = bv_last;
        if (a.w8) Bvh.sv = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(bv_last) + (size_t)W * a.Hd);
      } else {
        Bvh.p = static_cast<const uint8_t*>(a.Bv) + (size_t)h_ * W * a.Hd * (a.w8 ? 1 : 2);
      }
    }
    if (cf == cl) {
      finalize_out<W>(res, Bvh, outp, a.Hd, red, tid);
      return;
    }
    float* dst = a.partials + ((size_t)c + bh) * (W + 2);
    int* flag = reinterpret_cast<int*>(misc) + 8;
    if (tid == 0) *flag = (seen == cl - cf) ? 2 : 0;
    csync();
    const int early = *flag;
    if (tid < W + 2) {
      for (int e = tid; e < W + 2; e += kConsumerThreads) dst[e] = res[e];
      if (!early) __threadfence();  // publish before the counter bump
    }
    csync();
    if (!early) {
      if (tid == 0) {
        const int prev = atomicAdd(&a.counters[bh], 1);
        *flag = (prev == cl - cf) ? 1 : 0;
      }
      csync();
    }
    if (*flag) {
      if (!early) __threadfence();
      merge_rows<W, true>(a.partials + ((size_t)cf + bh) * (W + 2), cl - cf + 1, res, tid);
      if (tid == 0) atomicExch(&a.counters[bh], 0);
      finalize_out<W>(res, Bvh, outp, a.Hd, red, tid);
    }
  };

  int b, h, t;
  walk.locate(g_begin, b, h, t);
  int cb = -1, ch = -1;
  long long i = 0;
  for (long long g = g_begin; g < g_end; ++g, ++i) {
    if (b != cb || h != ch) {
      if (cb >= 0) end_segment(k - 1);
      const int sq = k % NQ;
      wait(&qready[sq], (uint32_t)((k / NQ) & 1));
      qst.step = ha->qstep[sq];
      if constexpr (CT::kScaled) {
        const uint32_t* pl = ha->planes[sq];
#pragma unroll
        for (int q = 0; q < QW; ++q) {
          qst.qh[q] = pl[(sub * 3 + 0) * QW + q];
          qst.qm[q] = pl[(sub * 3 + 1) * QW + q];
          qst.ql[q] = pl[(sub * 3 + 2) * QW + q];
        }
        if constexpr (CODEC == kCodecI4) {
          qst.ch = (int)pl[TPT * 3 * QW + sub * 3 + 0];
          qst.cm = (int)pl[TPT * 3 * QW + sub * 3 + 1];
          qst.cl = (int)pl[TPT * 3 * QW + sub * 3 + 2];
        }
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p)
          qst.qv[p] = make_float2(ha->qsv[sq][sub * VPT + 2 * p], ha->qsv[sq][sub * VPT + 2 * p + 1]);
      }
      if constexpr (C::kNSeg == 2) qst.swap_halves(swapped_lane(lane));
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfree[sq]);
#pragma unroll
      for (int p = 0; p < NP; ++p) acc[p] = make_float2(0.f, 0.f);
      m = kNegInf;
      l = 0.f;
      ++k;
      cb = b;
      ch = h;
    }
    const int s = (int)(i % S);
    // A timed-out wait only poisons the result (err is set); control flow stays
    // uniform so every consumer warp reaches every named barrier.
    wait(&full[s], (uint32_t)((i / S) & 1));
    process_tile<CODEC, VPT, TPT, NTOK>(stages + (size_t)s * C::kStageBytes, min(T, lens[b] - t * T), qst, m, l,
                                        acc, tid);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    walk.advance(b, h, t);
  }
  if (cb >= 0) finish_last(cb, ch);
}

// ------------------------------------------------------------------ cluster kernel (small problems)
// One thread-block cluster of `cluster` CTAs per (b, h) splits the cached
// tokens into contiguous chunks.  Each CTA issues its operand copies at
// launch and builds q' before it reads seq_lens (so under a programmatic
// dependent launch that work overlaps the preceding append), reduces its
// chunk to (m, l, o[W]) and stores it straight into a slot of the leader's
// shared memory with st.async stores whose bytes complete on the leader's
// mbarrier.  The leader merges the slots in rank order and writes out[b, h]
// with B_Vh staged in its shared memory: no global partials, counters or fences.
template <int CODEC, int VPT, int TPT, int NTOK, int QMODE>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_cluster_kernel(const DecodeArgs a) {
  using C = Cfg<CODEC, VPT, TPT, NTOK>;
  constexpr int T = C::kT, W = C::kW, S = C::kStages, NP = VPT / 2;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank(), csize = (int)cluster.num_blocks();
  const int h = blockIdx.y, b = blockIdx.z;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + S;
  uint64_t* segfull = empty + S;
  uint64_t* aux = segfull + 1;  // [0]: B_Vh staged (leader), [1]: slots filled (leader),
                                // [2]: pre-staged tile count known, [3]: tile total known
  float* qs = reinterpret_cast<float*>(smem + C::kOffQ);
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  float* res = reinterpret_cast<float*>(smem + C::kOffRes);
  float* misc = reinterpret_cast<float*>(smem + C::kOffMisc);
  uint32_t* planes = reinterpret_cast<uint32_t*>(smem + C::kOffParts);
  uint8_t* segbuf = smem + C::cluster_seg_off();
  float* slots = reinterpret_cast<float*>(segbuf + seg_bytes(QMODE, W, a.Hd));  // [csize][W + 2]
  __half* bvs = reinterpret_cast<__half*>(slots + (size_t)kMaxClusterSize * (W + 2));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Token chunk of this rank (multiple of 8 tokens, so scale copies stay aligned).
  const int chunk = ((a.L_cap + csize - 1) / csize + 7) & ~7;
  const int lo = min(a.L_cap, rank * chunk), hi = min(a.L_cap, lo + chunk);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(segfull, 1);
    mbar_init(&aux[0], 1);
    mbar_init(&aux[1], 1);
    mbar_init(&aux[2], 1);
    mbar_init(&aux[3], 1);
    fence_mbar_init();
    // leader: the other ranks' partial rows arrive as st.async transaction bytes
    if (rank == 0 && csize > 1) mbar_arrive_expect_tx(&aux[1], (uint32_t)((csize - 1) * (W + 2) * 4));
    // Operands first: they do not depend on the sequence length.
    const uint64_t keep = l2_evict_last_policy();
    issue_operands<W, QMODE>(segbuf, segfull, a, b, h, keep);
    if (rank == 0 && a.Bv != nullptr) {
      // B_Vh, and (int8 B_V) its column scales after it
      const uint32_t bb = (uint32_t)W * a.Hd * (a.w8 ? 1 : 2), sb = a.w8 ? (uint32_t)a.Hd * 4 : 0u;
      mbar_arrive_expect_tx(&aux[0], bb + sb);
      for (uint32_t off = 0; off < bb; off += 32768)
        bulk_g2s(reinterpret_cast<uint8_t*>(bvs) + off, static_cast<const uint8_t*>(a.Bv) + (size_t)h * bb + off,
                 min(32768u, bb - off), &aux[0], keep);
      if (a.w8) bulk_g2s(reinterpret_cast<uint8_t*>(bvs) + bb, a.sBv + (size_t)h * a.Hd, sb, &aux[0], keep);
    }
  }
  cluster_arrive_relaxed();  // barriers initialised; waited on before any remote access
  __syncthreads();           // barrier initialisation visible to every thread of this CTA

  // Per-stage valid rows, then (after the stages) the number of tiles staged
  // before the dependency wait and the total, for the consumers.  red[] is
  // free until the final reduction; the producer's last write to it precedes
  // the last tile's arrive.
  int* tile_info = reinterpret_cast<int*>(red);

  // Everything above reads only q and the B matrices.  The tiles are the fixed
  // grid [lo + i T, lo + (i + 1) T) of this rank's rows below the length.
  // Behind the append that writes this step's row and seq_lens (programmatic
  // dependent launch, dep 2) the producer stages, before it waits, the rows
  // that append cannot touch: it writes only row seq_lens[b] as it was at
  // launch, and the value read here is that one or the advanced one, so rows
  // below it minus one are final either way.  A tile straddling that bound is
  // filled in two parts (its barrier completes only with the second part).
  // The grid, and so the arithmetic, does not depend on that early read.
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      using CT = typename C::CT;
      const uint64_t pol = l2_evict_first_policy();
      bool ok = true;
      // rows [r0 + off, r0 + off + n) of the tile at r0 into stage st, completing on bar
      auto copy_rows = [&](uint8_t* st, int r0, int off, int n, uint64_t* bar) {
        const int rr = r0 + off;
        const size_t head_row = ((size_t)b * a.H + h) * a.L_cap + rr;
        const size_t row0 = a.heads_share ? (size_t)b * a.L_cap + rr : head_row;
        const uint32_t cbytes = (uint32_t)n * C::kRB;
        const uint32_t sbytes = CT::kScaled ? (uint32_t)((n + 7) & ~7) * 2u : 0u;
        bulk_g2s(st + (size_t)off * C::kRB, a.lat_k + row0 * C::kRB, cbytes, bar, pol);
        bulk_g2s(st + C::kCodeBytes + (size_t)off * C::kRB, a.lat_v + row0 * C::kRB, cbytes, bar, pol);
        if (CT::kScaled) {
          bulk_g2s(st + 2 * C::kCodeBytes + off * 2, a.scale_k + head_row, sbytes, bar, pol);
          bulk_g2s(st + 2 * C::kCodeBytes + C::kScaleBytes + off * 2, a.scale_v + head_row, sbytes, bar, pol);
        }
      };
      auto tile_bytes = [&](int n) {
        return 2u * (uint32_t)n * C::kRB + (CT::kScaled ? 4u * (uint32_t)((n + 7) & ~7) : 0u);
      };
      auto claim = [&](int i) {  // stage of tile i, free for reuse
        const int s = i % S;
        if (i >= S && !mbar_wait_bounded(&empty[s], (uint32_t)(((i / S) - 1) & 1))) {
          set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
          ok = false;
        }
        return s;
      };
      int pre_end = lo;
      if (a.dep == 2) {
        const int v = clamp_len(ld_relaxed_gpu(a.seq_lens + b), a.L_cap);
        pre_end = max(lo, min(hi, v - 1) & ~7);
      }
      if (a.dep == 2 && hi > lo && pre_end == hi) {
        // Every row of this rank lies below the bound: the rows are final and
        // the final length is above hi whichever value the early read saw, so
        // the tiles, their counts and their arithmetic are those of the plain
        // decode; they are handed over without waiting for the append.  The
        // leader still waits before it exits, so the grid never completes
        // before the grid it was launched behind.
        const int total = (hi - lo + T - 1) / T;
        tile_info[S] = total;
        mbar_arrive(&aux[2]);
        for (int i = 0; i < total && ok; ++i) {
          const int s = claim(i);
          if (!ok) break;
          const int n = min(T, hi - (lo + i * T));
          tile_info[s] = n;
          mbar_arrive_expect_tx(&full[s], tile_bytes(n));
          copy_rows(stages + (size_t)s * C::kStageBytes, lo + i * T, 0, n, &full[s]);
        }
        tile_info[S + 1] = total;
        mbar_arrive(&aux[3]);
        if (rank == 0) {
          griddep_wait();
          const int raw = a.seq_lens[b];
          if ((raw < 0 || raw > a.L_cap) && h == 0) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
        }
        const int issued = ok ? total : 0;
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          if (!mbar_wait_bounded(&full[i % S], (uint32_t)((i / S) & 1))) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
        if (!mbar_wait_bounded(segfull, 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
        if (rank == 0 && a.Bv != nullptr && !mbar_wait_bounded(&aux[0], 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      } else {
        const int npre = (pre_end - lo) / T, part = (pre_end - lo) % T;  // whole tiles below the bound, rows of the next
        tile_info[S] = npre;
        mbar_arrive(&aux[2]);
        for (int i = 0; i < npre && ok; ++i) {
          const int s = claim(i);
          if (!ok) break;
          tile_info[s] = T;
          mbar_arrive_expect_tx(&full[s], tile_bytes(T));
          copy_rows(stages + (size_t)s * C::kStageBytes, lo + i * T, 0, T, &full[s]);
        }
        if (ok && part > 0) {
          const int s = claim(npre);
          if (ok) {
            mbar_expect_tx(&full[s], tile_bytes(part));  // no arrive yet: the rest follows after the wait
            copy_rows(stages + (size_t)s * C::kStageBytes, lo + npre * T, 0, part, &full[s]);
          }
        }
        griddep_wait();
        const int raw = a.seq_lens[b];
        if ((raw < 0 || raw > a.L_cap) && rank == 0 && h == 0) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
        const int end = max(pre_end, min(hi, clamp_len(raw, a.L_cap)));  // pre_end <= end holds by construction
        const int total = end > lo ? (end - lo + T - 1) / T : 0;         // > npre whenever part > 0
        tile_info[S + 1] = total;
        mbar_arrive(&aux[3]);
        for (int i = npre; i < total && ok; ++i) {
          const int r0 = lo + i * T, n = min(T, end - r0);
          const bool split = (i == npre && part > 0);
          const int s = split ? i % S : claim(i);  // a split tile's stage was claimed before the wait
          if (!ok) break;
          tile_info[s] = n;
          const int off = split ? part : 0;
          mbar_arrive_expect_tx(&full[s], n > off ? tile_bytes(n) - tile_bytes(off) : 0u);
          if (n > off) copy_rows(stages + (size_t)s * C::kStageBytes, r0, off, n - off, &full[s]);
        }
        const int issued = ok ? total : 0;
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          if (!mbar_wait_bounded(&full[i % S], (uint32_t)((i / S) & 1))) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
        if (!mbar_wait_bounded(segfull, 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
        if (rank == 0 && a.Bv != nullptr && !mbar_wait_bounded(&aux[0], 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      }
    }
    cluster_wait();
    return;
  }

  // consumers: every staged tile reaches them through the producer, which
  // waits on the preceding grid before staging anything that grid may write.
  const int sub = tid % TPT;
  QState<CODEC, VPT> qst;
  float2 acc[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) acc[p] = make_float2(0.f, 0.f);
  float m = kNegInf, l = 0.f;
  bool timed_out = false;
  auto cwait = [&](uint64_t* bar, uint32_t parity) {
    if (!mbar_wait_bounded(bar, parity, timed_out ? 0ull : kWaitLimitNs)) {
      if (!timed_out && lane == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      timed_out = true;
    }
  };
  cwait(segfull, 0);
  build_query<CODEC, VPT, W, QMODE>(qst, segbuf, qs, misc, planes, a, tid, sub);
  const int max_tiles = (hi - lo + T - 1) / T;
  cwait(&aux[2], 0);
  const int npre = timed_out ? 0 : min(tile_info[S], max_tiles);
  int total = -1;
  for (int i = 0; i < max_tiles; ++i) {
    if (i >= npre) {
      if (total < 0) {
        cwait(&aux[3], 0);
        total = timed_out ? 0 : min(tile_info[S + 1], max_tiles);
      }
      if (i >= total) break;
    }
    const int s = i % S;
    cwait(&full[s], (uint32_t)((i / S) & 1));
    if (timed_out) break;
    process_tile<CODEC, VPT, TPT, NTOK>(stages + (size_t)s * C::kStageBytes, tile_info[s], qst, m, l, acc, tid);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  csync();  // every consumer has read its last tile_info before red[] is reused
  reduce_to_res<VPT, TPT, W, C::kNSeg>(m, l, acc, red, res, tid);

  cluster_wait();  // every CTA of the cluster has initialised its barriers
  if (rank != 0) {
    // Partial row straight into the leader's slot; each store completes its
    // bytes on the leader's barrier (no fence, no separate arrive).
    const uint32_t rslot = mapa_shared(slots + (size_t)rank * (W + 2), 0), rbar = mapa_shared(&aux[1], 0);
    for (int e = tid; e < W + 2; e += kConsumerThreads) st_async_f32(rslot + 4u * e, res[e], rbar);
    return;
  }
  if (csize > 1) {
    for (int e = tid; e < W + 2; e += kConsumerThreads) slots[e] = res[e];
    if (tid == 0 && !mbar_wait_cluster_bounded(&aux[1], 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    csync();
    merge_rows<W, false>(slots, csize, res, tid);
  }
  BvRef Bvh{nullptr, a.w8, nullptr};
  if (a.Bv != nullptr) {
    if (!mbar_wait_bounded(&aux[0], 0, timed_out ? 0ull : kWaitLimitNs) && lane == 0)
      set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    Bvh.p = bvs;
    if (a.w8) Bvh.sv = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(bvs) + (size_t)W * a.Hd);
  }
  finalize_out<W>(res, Bvh, a.out + ((size_t)b * a.H + h) * a.Hd, a.Hd, red, tid);
}

// ------------------------------------------------------------------ one-kernel step (one sequence)
// The latent append and the decode of one step in one grid, for a single
// sequence (B = 1) whose decode takes the cluster path with the append's
// cluster size and at most one tile per rank.  Cluster h does head h's append
// for K and V (rank q projects its E slice [q Ec, (q + 1) Ec), as the append
// kernel's rank q) and head h's decode (rank q its token chunk, as the
// cluster decode's rank q).  The append's partial rows go to the rank whose
// chunk holds the new row (the owner) rather than to rank 0: the owner sums
// them in rank order, quantises, writes the row to the cache and into its
// staged tile, and adds that token to its softmax state after the tile's
// other rows.  With one token per lane and tile, a lane's state after the two
// passes is the one a single pass gives.  The owner also merges the ranks'
// decode partials (in rank order, as rank 0 of the cluster decode does) and
// writes out[h].  So every output equals that of the append kernel followed
// by the cluster decode, bit for bit.
//
// Order of work.  Producer lane: barriers, then bulk copies of B_Kh, the
// query (and, for int8 B, B_K's column scales) and of this rank's A_Kh and
// A_Vh slices (contiguous blocks, four chunks each with a barrier apiece;
// behind a grid that writes the query, the query comes after the dependency
// wait).  Then the length (its load overlaps the issue), which reaches the
// consumers through an mbarrier; B_Vh (and its int8 column scales) into the
// merging rank; and, once the slices have landed, the cached rows of the
// chunk below the new row.  Consumers: q' and the x slice rotation while the
// copies land (warps 0 and 1 load the int8 A column scales they would need
// as quantisers); the K and V projections of the slice chunk by chunk,
// reduced across the CTA in one pass and stored into the owner's slots; the
// old rows; the owner quantises and processes the new row; every rank but the
// merging one sends its decode partial there, which merges and writes out[h].
// The latent width is a compile-time constant (r == W; the host checks it).
//
// The length advance: each CTA's producer lane, after its read of seq_lens,
// counts the CTA in the append's completion counter (acq_rel); the last of
// the grid's CTAs stores the advanced length and resets the counter.
constexpr int kStepChunks = 4;  // A slice chunks per unit, each with its own barrier
struct StepLayout {
  size_t slice_k, slice_v, xs, slots, red, bar, pos, total;
};
__host__ __device__ inline StepLayout step_layout(size_t base, int Ec, int r, int w8, int csize) {
  auto up = [](size_t v, size_t a) { return (v + a - 1) / a * a; };
  StepLayout L;
  const size_t sb = (size_t)Ec * r * (w8 ? 1 : 2);
  size_t o = up(base, 128);
  L.slice_k = o;
  o = up(o + sb, 128);
  L.slice_v = o;
  o = up(o + sb, 128);
  L.xs = o;
  o = up(o + (size_t)Ec * 4, 16);
  L.slots = o;  // [csize][K, V][r]
  o = up(o + (size_t)csize * 2 * r * 4, 16);
  L.red = o;
  o = up(o + (size_t)kAppendWarps * 2 * r * 4, 16);
  L.bar = o;
  o += (2 * kStepChunks + 2) * 8;
  L.pos = o;
  o += 16;
  L.total = up(o, 128);
  return L;
}

template <int CODEC, int VPT, int TPT, bool W8>
__global__ void __launch_bounds__(kDecodeThreads, 2) step_cluster_kernel(const DecodeArgs a, const AppendArgs ap) {
  using C = Cfg<CODEC, VPT, TPT, 1, 1>;
  constexpr int W = C::kW, NP = VPT / 2;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank(), csize = (int)cluster.num_blocks();
  const int h = blockIdx.y;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stage = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* segfull = full + 2;  // (full[1], empty[1], segfull, aux[4]) as in the cluster decode
  uint64_t* aux = segfull + 1;   // [0]: B_Vh staged, [1]: decode partials landed (merging rank)
  float* qs = reinterpret_cast<float*>(smem + C::kOffQ);
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  float* res = reinterpret_cast<float*>(smem + C::kOffRes);
  float* misc = reinterpret_cast<float*>(smem + C::kOffMisc);
  uint32_t* planes = reinterpret_cast<uint32_t*>(smem + C::kOffParts);
  uint8_t* segbuf = smem + C::cluster_seg_off();
  float* slots = reinterpret_cast<float*>(segbuf + seg_bytes(kQProj, W, a.Hd));  // [csize][W + 2]
  __half* bvs = reinterpret_cast<__half*>(slots + (size_t)kMaxClusterSize * (W + 2));

  constexpr int r = W;  // the latent width (the host launches this kernel only when r == W)
  const int E = ap.E, Ec = E / csize, e0 = rank * Ec;
  const StepLayout L = step_layout(C::cluster_smem_bytes(kQProj, a.Hd), Ec, r, W8, csize);
  uint8_t* slice_k = smem + L.slice_k;
  uint8_t* slice_v = smem + L.slice_v;
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  float* aslots = reinterpret_cast<float*>(smem + L.slots);
  float* ared = reinterpret_cast<float*>(smem + L.red);
  // [u * kStepChunks + c]: chunk c of slice u landed; then the ranks' partial
  // rows landed (owner), and the length known
  uint64_t* abar = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* bar_part = abar + 2 * kStepChunks;
  uint64_t* bar_pos = bar_part + 1;
  int* pos_sm = reinterpret_cast<int*>(smem + L.pos);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = ((a.L_cap + csize - 1) / csize + 7) & ~7;
  const int lo = min(a.L_cap, rank * chunk), hi = min(a.L_cap, lo + chunk);
  const uint32_t piece = (uint32_t)Ec * r * (W8 ? 1 : 2) / kStepChunks;  // bytes per slice chunk
  const int piece_rows = Ec / kStepChunks;

  if (tid == kConsumerThreads) {
    mbar_init(&full[0], 1);
    mbar_init(segfull, 1);
    mbar_init(&aux[0], 1);
    mbar_init(&aux[1], 1);
    for (int i = 0; i < 2 * kStepChunks + 2; ++i) mbar_init(&abar[i], 1);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();  // barriers initialised; waited on before any remote access
  __syncthreads();

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const int pos = ld_relaxed_gpu(ap.seq_lens);  // consumed below: the copies are issued meanwhile
      const uint64_t keep = l2_evict_last_policy(), once = l2_evict_first_policy();
      const uint32_t bb = (uint32_t)W * a.Hd * (a.w8 ? 1 : 2), qb = (uint32_t)a.Hd * 2;
      const uint16_t* qh = static_cast<const uint16_t*>(a.q) + (size_t)h * a.Hd;
      const uint32_t sb = a.w8 ? (uint32_t)a.Hd * 4 : 0u;  // int8 B_K / B_V: their column scales
      mbar_arrive_expect_tx(segfull, bb + qb + sb);
      bulk_g2s(segbuf, static_cast<const uint8_t*>(a.Bk) + (size_t)h * bb, bb, segfull, keep);
      if (a.w8) bulk_g2s(segbuf + bb + qb, a.sBk + (size_t)h * a.Hd, sb, segfull, keep);
      if (!ap.dep) bulk_g2s(segbuf + bb, qh, qb, segfull, keep);
      for (int u = 0; u < 2; ++u) {
        const uint8_t* src = static_cast<const uint8_t*>(u ? ap.Av : ap.Ak) + ((size_t)h * E + e0) * r * (W8 ? 1 : 2);
        uint8_t* dst = u ? slice_v : slice_k;
        for (int c = 0; c < kStepChunks; ++c) {
          mbar_arrive_expect_tx(&abar[u * kStepChunks + c], piece);
          bulk_g2s(dst + (size_t)c * piece, src + (size_t)c * piece, piece, &abar[u * kStepChunks + c], once);
        }
      }
      if (ap.dep) {
        griddep_wait();  // the query is written by the preceding grid
        bulk_g2s(segbuf + bb, qh, qb, segfull, keep);
      }
      const bool ok = pos >= 0 && pos < a.L_cap;
      const int lead = ok ? pos / chunk : 0;                   // the owner, which also merges
      const int len_old = ok ? pos : clamp_len(pos, a.L_cap);  // rows final before the step
      const int n_old = max(0, min(hi, len_old) - lo);          // of them in this rank's chunk
      if (rank == lead && csize > 1) {
        // the other ranks' partial rows (some may have landed already)
        if (ok) mbar_arrive_expect_tx(bar_part, (uint32_t)((csize - 1) * 2 * r * 4));
        mbar_arrive_expect_tx(&aux[1], (uint32_t)((csize - 1) * (W + 2) * 4));
      }
      *pos_sm = pos;
      mbar_arrive(bar_pos);
      if (rank == lead) {
        mbar_arrive_expect_tx(&aux[0], bb + sb);
        for (uint32_t off = 0; off < bb; off += 32768)
          bulk_g2s(reinterpret_cast<uint8_t*>(bvs) + off, static_cast<const uint8_t*>(a.Bv) + (size_t)h * bb + off,
                   min(32768u, bb - off), &aux[0], keep);
        if (a.w8) bulk_g2s(reinterpret_cast<uint8_t*>(bvs) + bb, a.sBv + (size_t)h * a.Hd, sb, &aux[0], keep);
      }
      // The cached rows are read after this CTA's A slices have landed: they
      // are needed only after the projection, and would compete with it for
      // HBM bandwidth.
      bool done = true;
      for (int i = 0; i < 2 * kStepChunks; ++i) done = mbar_wait_bounded(&abar[i], 0) && done;
      if (n_old > 0) {
        const size_t row0 = (size_t)h * a.L_cap + lo;
        const uint32_t cbytes = (uint32_t)n_old * C::kRB, sbytes = (uint32_t)((n_old + 7) & ~7) * 2u;
        mbar_arrive_expect_tx(&full[0], 2 * cbytes + 2 * sbytes);
        bulk_g2s(stage, a.lat_k + row0 * C::kRB, cbytes, &full[0], once);
        bulk_g2s(stage + C::kCodeBytes, a.lat_v + row0 * C::kRB, cbytes, &full[0], once);
        bulk_g2s(stage + 2 * C::kCodeBytes, a.scale_k + row0, sbytes, &full[0], once);
        bulk_g2s(stage + 2 * C::kCodeBytes + C::kScaleBytes, a.scale_v + row0, sbytes, &full[0], once);
      } else {
        mbar_arrive(&full[0]);
      }
      if (ok) {
        // This CTA's read of the length is complete (its value was used above).
        const int prev = atom_add_acq_rel_gpu(ap.counter, 1);
        if (prev == (int)(gridDim.x * gridDim.y) - 1) {
          st_relaxed_gpu(ap.seq_lens, pos + 1);
          st_relaxed_gpu(ap.counter, 0);
        }
      }
      // No copy may still be landing when the CTA exits (the consumers may have
      // given up on a barrier).
      done = mbar_wait_bounded(&full[0], 0) && mbar_wait_bounded(segfull, 0) && done;
      if (rank == lead) done = mbar_wait_bounded(&aux[0], 0) && done;
      if (!done) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    }
    cluster_wait();
    return;
  }

  // ---- consumers
  bool timed_out = false;
  auto cwait = [&](uint64_t* bar, uint32_t parity, bool cluster_scope) {
    const uint64_t lim = timed_out ? 0ull : kWaitLimitNs;
    const bool got = cluster_scope ? mbar_wait_cluster_bounded(bar, parity, lim) : mbar_wait_bounded(bar, parity, lim);
    if (!got) {
      if (!timed_out && lane == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      timed_out = true;
    }
  };
  auto consumer_sync = []() { csync(); };
  // int8 weights: warps 0 and 1 (the quantisers of K and V, should this rank
  // own the new row) load their column scales now.
  ColScales<W> cs;
  if (W8 && warp < 2) cs.load((warp ? ap.sAv : ap.sAk) + (size_t)h * r, r, lane);
  // x slice of the append (registers on the fast path)
  const bool fast = x_fast_path(1, Ec, ap.blk);
  uint2 xraw[kXChunks];
  if (ap.dep) griddep_wait();  // x is written by the preceding grid
  if (fast) load_x_slice(xraw, ap.x, 1, E, e0, Ec, warp, lane);

  // q' and its byte planes, the rotated x slice
  const int sub = tid % TPT;
  QState<CODEC, VPT> qst;
  cwait(segfull, 0, false);
  build_query<CODEC, VPT, W, kQProj>(qst, segbuf, qs, misc, planes, a, tid, sub);
  rotate_x_slice(fast, xraw, xs, ap.x, ap.x_dtype, 1, E, e0, Ec, ap.blk, tid, consumer_sync);

  cwait(bar_pos, 0, false);
  const int pos = timed_out ? -1 : *pos_sm;
  const bool ok = pos >= 0 && pos < a.L_cap;
  const int lead = ok ? pos / chunk : 0;
  const bool own = ok && rank == lead;
  const int len_old = ok ? pos : clamp_len(pos, a.L_cap);
  const int n_old = max(0, min(hi, len_old) - lo);
  if (!ok && rank == 0 && h == 0 && tid == 0) {
    set_err(a.err, WSVD_DEVERR_CACHE_FULL);
    if (pos < 0 || pos > a.L_cap) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
  }
  cluster_wait();  // every CTA of the cluster has initialised its barriers

  // the append: K and V projections of this rank's E slice, chunk by chunk,
  // reduced in one pass into the owner's slots [rank][K, V]
  if (ok) {
    const int ncg = r / 8, nrg = kAppendThreads / ncg, rg = tid / ncg, cgi = tid % ncg;
    const int nrows = rg < Ec ? (Ec - 1 - rg) / nrg + 1 : 0;
    float2 cacc[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
#pragma unroll
      for (int k = 0; k < 4; ++k) cacc[u][k] = make_float2(0.f, 0.f);
      const uint8_t* sl = u ? slice_v : slice_k;
      float2 (&cu)[1][4] = *reinterpret_cast<float2 (*)[1][4]>(&cacc[u][0]);
      int landed = 0, bound = 0;  // chunks of this slice known to have landed; rows below bound are in
      for (int k = 0, e = rg; k < nrows; ++k, e += nrg) {
        while (e >= bound) {
          cwait(&abar[u * kStepChunks + landed++], 0, false);
          bound += piece_rows;
        }
        uint4 av;
        if (W8) {
          const uint2 v2 = *reinterpret_cast<const uint2*>(sl + (size_t)e * r + cgi * 8);
          av = make_uint4(v2.x, v2.y, 0u, 0u);
        } else {
          av = *reinterpret_cast<const uint4*>(sl + ((size_t)e * r + cgi * 8) * 2);
        }
        accumulate_row<1, W8>(av, xs, 1, 0, Ec, e, cu);
      }
    }
    const bool remote = rank != lead;
    float* dst = aslots + (size_t)rank * 2 * r;
    reduce_cta<2, W / 8>(cacc, W, 2, ared, dst, remote ? mapa_shared(dst, lead) : 0u,
                         remote ? mapa_shared(bar_part, lead) : 0u, tid, consumer_sync);
  }

  // the rows of the chunk that precede the new one
  float2 acc[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) acc[p] = make_float2(0.f, 0.f);
  float m = kNegInf, l = 0.f;
  cwait(&full[0], 0, false);
  if (n_old > 0 && !timed_out) process_tile<CODEC, VPT, TPT, 1>(stage, n_old, qst, m, l, acc, tid);

  if (own) {
    // quantise the new row (warp 0: K, warp 1: V) into the cache and the staged tile
    const int t = pos - lo;
    if (warp < 2) {
      const int u = warp;
      if (csize > 1) cwait(bar_part, 0, true);
      const size_t row = (size_t)h * a.L_cap + pos;
      const int RB = r * ap.bits / 8;
      uint8_t* tile_codes = stage + (size_t)u * C::kCodeBytes + (size_t)t * C::kRB;
      const __half sh = quantise_append_row<W8, W>(aslots + (size_t)u * r, (size_t)2 * r, csize, r, ap.bits, ap.hnorm,
                                                   cs, true, (u ? ap.lat_v : ap.lat_k) + row * RB, tile_codes, lane);
      if (lane == 0) {
        (u ? ap.scale_v : ap.scale_k)[row] = sh;
        reinterpret_cast<__half*>(stage + 2 * C::kCodeBytes + (size_t)u * C::kScaleBytes)[t] = sh;
      }
    }
    csync();  // the new row is in the tile
    // Only the warp holding the new token's lanes has a valid token in this
    // pass; the other lanes' states would not change.
    if (!timed_out && warp == (t * TPT) / 32) process_tile<CODEC, VPT, TPT, 1>(stage, t + 1, qst, m, l, acc, tid, t);
  }
  reduce_to_res<VPT, TPT, W, C::kNSeg>(m, l, acc, red, res, tid);
  if (rank != lead) {
    // Partial row straight into the merging rank's slot; each store completes
    // its bytes on that rank's barrier.
    const uint32_t rslot = mapa_shared(slots + (size_t)rank * (W + 2), lead), rbar = mapa_shared(&aux[1], lead);
    for (int e = tid; e < W + 2; e += kConsumerThreads) st_async_f32(rslot + 4u * e, res[e], rbar);
    return;
  }

  // the merging rank: the ranks' partials in rank order, up-projected through B_Vh
  if (csize > 1) {
    for (int e = tid; e < W + 2; e += kConsumerThreads) slots[(size_t)rank * (W + 2) + e] = res[e];
    if (tid == 0 && !mbar_wait_cluster_bounded(&aux[1], 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    csync();
    merge_rows<W, false>(slots, csize, res, tid);
  }
  if (!mbar_wait_bounded(&aux[0], 0, timed_out ? 0ull : kWaitLimitNs) && lane == 0)
    set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
  const BvRef Bvh{bvs, a.w8,
                  a.w8 ? reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(bvs) + (size_t)W * a.Hd)
                       : nullptr};
  finalize_out<W>(res, Bvh, a.out + (size_t)h * a.Hd, a.Hd, red, tid);
}

// ------------------------------------------------------------------ host side
namespace {

// Per-device caches of the host-side launch set-up (SM count, occupancy, the
// dynamic shared-memory opt-in), so a decode call is one launch and no
// repeated driver queries.
struct HostCache {
  std::mutex mu;
  std::map<std::pair<const void*, int>, size_t> smem_optin;  // (kernel, device) -> bytes opted in
  std::map<std::tuple<const void*, int, size_t>, int> occ;   // (kernel, device, smem) -> CTAs per SM
  std::map<int, int> sms;                                    // device -> SM count
};
HostCache& host_cache() {
  static HostCache c;
  return c;
}

cudaError_t ensure_smem(const void* fn, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  HostCache& c = host_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  auto key = std::make_pair(fn, dev);
  auto it = c.smem_optin.find(key);
  if (it != c.smem_optin.end() && it->second >= smem) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) c.smem_optin[key] = smem;
  return e;
}

int device_sms_and_occupancy(const void* fn, size_t smem, int threads, int* occ_out) {
  int dev = 0, sms = 148, occ = 1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *occ_out = 1;
    return sms;
  }
  HostCache& c = host_cache();
  {
    std::lock_guard<std::mutex> lock(c.mu);
    auto s = c.sms.find(dev);
    auto o = c.occ.find(std::make_tuple(fn, dev, smem));
    if (s != c.sms.end() && o != c.occ.end()) {
      *occ_out = o->second;
      return s->second;
    }
  }
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (ensure_smem(fn, smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess || occ < 1)
    occ = 1;
  std::lock_guard<std::mutex> lock(c.mu);
  c.sms[dev] = sms;
  c.occ[std::make_tuple(fn, dev, smem)] = occ;
  *occ_out = occ;
  return sms;
}

struct KernelInfo {
  const void* fn;          // persistent kernel
  const void* cfn;         // cluster kernel (same tile shape), or null
  int pqmode;              // query mode of the persistent kernel
  size_t (*smem)(int B, int qmode, int Hd);
  size_t (*csmem)(int qmode, int Hd);
  int tile;
};

constexpr int kNoCluster = -1;

// PQ: query mode of the persistent kernel; CQ: of the cluster kernel (or
// kNoCluster).  The low-rank codecs project q' inside the cluster kernel but
// take it precomputed (kQGlobal) in the persistent one, whose helper warp
// then only packs byte planes.
template <int CODEC, int VPT, int TPT, int NTOK, int PQ, int CQ>
KernelInfo info() {
  using C = Cfg<CODEC, VPT, TPT, NTOK>;
  const void* cfn = nullptr;
  if constexpr (CQ != kNoCluster) cfn = reinterpret_cast<const void*>(&decode_cluster_kernel<CODEC, VPT, TPT, NTOK, CQ>);
  return KernelInfo{reinterpret_cast<const void*>(&decode_kernel<CODEC, VPT, TPT, NTOK, PQ>), cfn, PQ,
                    &C::smem_bytes, &C::cluster_smem_bytes, C::kT};
}

// Instantiated shapes.  `big` selects the variant with more tokens per lane per
// tile (fewer, larger tiles) for long caches.  qmode is the caller's: kQProj
// (low-rank), kQDirect (dense) or kQGlobal (shared latent).
bool pick(int codec, int rowbytes, int qmode, bool big, KernelInfo* ki) {
  constexpr int P = kQGlobal, X = kQProj;
  if (qmode == kQProj && codec == kCodecI8) {
    switch (rowbytes) {
      case 16: *ki = big ? info<kCodecI8, 16, 1, 4, P, X>() : info<kCodecI8, 16, 1, 2, P, X>(); return true;
      case 32: *ki = big ? info<kCodecI8, 32, 1, 2, P, X>() : info<kCodecI8, 32, 1, 1, P, X>(); return true;
      case 64: *ki = info<kCodecI8, 32, 2, 1, P, X>(); return true;
      case 128: *ki = info<kCodecI8, 32, 4, 1, P, X>(); return true;
    }
  } else if (qmode == kQProj && codec == kCodecI4) {
    switch (rowbytes) {
      case 16: *ki = big ? info<kCodecI4, 32, 1, 2, P, X>() : info<kCodecI4, 32, 1, 1, P, X>(); return true;
      case 32: *ki = info<kCodecI4, 32, 2, 1, P, X>(); return true;
      case 64: *ki = info<kCodecI4, 32, 4, 1, P, X>(); return true;
    }
  } else if (qmode == kQDirect && codec == kCodecF16) {
    switch (rowbytes) {
      case 64: *ki = info<kCodecF16, 16, 2, 2, kQDirect, kQDirect>(); return true;
      case 128: *ki = info<kCodecF16, 16, 4, 2, kQDirect, kQDirect>(); return true;
      case 256: *ki = info<kCodecF16, 16, 8, 2, kQDirect, kQDirect>(); return true;
      case 512: *ki = info<kCodecF16, 16, 16, 2, kQDirect, kQDirect>(); return true;
    }
  } else if (qmode == kQGlobal && codec == kCodecF16) {
    switch (rowbytes) {
      case 256: *ki = info<kCodecF16, 16, 8, 2, P, kNoCluster>(); return true;
      case 512: *ki = info<kCodecF16, 16, 16, 2, P, kNoCluster>(); return true;
      case 1024: *ki = info<kCodecF16, 16, 32, 1, P, kNoCluster>(); return true;
      case 2048: *ki = info<kCodecF16, 32, 32, 1, P, kNoCluster>(); return true;
    }
  }
  return false;
}

// The launch plan of one decode call: the cluster kernel (few tiles per
// resident CTA, B_Vh fits in the leader's shared memory) or the persistent
// grid, large-tile variant when there are several tiles per resident CTA.
struct Plan {
  bool cluster;
  int csize;        // cluster path: CTAs per (b, h)
  KernelInfo ki;    // the kernel to launch
  size_t smem;
  int ctas;         // persistent path: grid size
};

bool plan_decode(int codec, int rowbytes, int qmode, const DecodeArgs& a, Plan* pl) {
  KernelInfo small, big;
  if (!pick(codec, rowbytes, qmode, false, &small) || !pick(codec, rowbytes, qmode, true, &big)) return false;
  int occ = 1;
  const size_t smem_small = small.smem(a.B, small.pqmode, a.Hd);
  const int sms = device_sms_and_occupancy(small.fn, smem_small, kPersistThreads, &occ);
  const long long resident = (long long)sms * occ;
  const long long tiles_small = (long long)a.B * a.H * ((a.L_cap + small.tile - 1) / small.tile);
  const size_t csmem = small.cfn ? small.csmem(qmode, a.Hd) : 0;
  if (small.cfn && tiles_small <= 2 * resident && csmem <= 112 * 1024 && a.H <= 65535) {
    pl->cluster = true;
    pl->csize = (int)std::min<long long>(kMaxClusterSize, std::max(1, (a.L_cap + 127) / 128));
    pl->ki = small;
    pl->smem = csmem;
    pl->ctas = 0;
    return true;
  }
  const size_t smem_big = big.smem(a.B, big.pqmode, a.Hd);
  device_sms_and_occupancy(big.fn, smem_big, kPersistThreads, &occ);
  const long long tiles_big = (long long)a.B * a.H * ((a.L_cap + big.tile - 1) / big.tile);
  const KernelInfo& ki = (tiles_big >= 4 * (long long)sms * occ) ? big : small;
  const size_t smem = ki.smem(a.B, ki.pqmode, a.Hd);
  device_sms_and_occupancy(ki.fn, smem, kPersistThreads, &occ);
  const long long tiles_max = (long long)a.B * a.H * ((a.L_cap + ki.tile - 1) / ki.tile);
  long long ctas = (long long)sms * occ;
  if (ctas > tiles_max) ctas = tiles_max;
  if (ctas > kMaxDecodeCtas) ctas = kMaxDecodeCtas;
  if (ctas < 1) ctas = 1;
  pl->cluster = false;
  pl->csize = 0;
  pl->ki = ki;
  pl->smem = smem;
  pl->ctas = (int)ctas;
  return true;
}


// ---- one-kernel step: instantiated shapes (one token per lane and tile, r = 32)
using StepFn = void (*)(const DecodeArgs, const AppendArgs);
struct StepInfo {
  StepFn fn;
  int tile, rb;
  size_t (*base)(int qmode, int Hd);  // the cluster decode's part of the shared memory
};
template <int CODEC, int VPT, int TPT, bool W8>
StepInfo step_info() {
  using C = Cfg<CODEC, VPT, TPT, 1, 1>;
  return StepInfo{&step_cluster_kernel<CODEC, VPT, TPT, W8>, C::kT, C::kRB, &C::cluster_smem_bytes};
}
bool pick_step(int codec, int rowbytes, bool w8, StepInfo* si) {
  if (codec == kCodecI8 && rowbytes == 32) {
    *si = w8 ? step_info<kCodecI8, 32, 1, true>() : step_info<kCodecI8, 32, 1, false>();
    return true;
  }
  if (codec == kCodecI4 && rowbytes == 16) {
    *si = w8 ? step_info<kCodecI4, 32, 1, true>() : step_info<kCodecI4, 32, 1, false>();
    return true;
  }
  return false;
}
struct StepPlan {
  StepInfo si;
  int csize;
  size_t smem;
};
// The one-kernel step applies to one sequence whose decode takes the cluster
// path with the append's cluster size, each rank's chunk within one tile, and
// a shared-memory footprint that leaves two CTAs per SM.
bool plan_step(const AppendArgs& ap, const DecodeArgs& a, StepPlan* sp) {
  if (ap.B != 1 || a.B != 1 || a.H != ap.H || a.W != ap.r || a.L_cap != ap.L_cap || a.L_cap < 8 || a.H > 65535)
    return false;
  const int codec = ap.bits == 8 ? kCodecI8 : kCodecI4, rowbytes = ap.r * ap.bits / 8;
  if (!pick_step(codec, rowbytes, ap.w8 != 0, &sp->si) || sp->si.rb != rowbytes || a.w8 != ap.w8) return false;
  Plan pl;
  if (!plan_decode(codec, rowbytes, kQProj, a, &pl) || !pl.cluster || pl.csize != ap.cluster) return false;
  const int cs = ap.cluster;
  const int chunk = ((a.L_cap + cs - 1) / cs + 7) & ~7;
  if (chunk > sp->si.tile) return false;
  sp->csize = cs;
  sp->smem = step_layout(sp->si.base(kQProj, a.Hd), ap.E / cs, ap.r, ap.w8, cs).total;
  return sp->smem <= 113 * 1024;
}
}  // namespace

bool decode_supported(int codec, int rowbytes, int qmode) {
  KernelInfo ki;
  return pick(codec, rowbytes, qmode, false, &ki) && pick(codec, rowbytes, qmode, true, &ki);
}

int decode_launch_count(int codec, int rowbytes, int qmode, const DecodeArgs& a) {
  Plan pl;
  if (!plan_decode(codec, rowbytes, qmode, a, &pl)) return 0;
  return (!pl.cluster && pl.ki.pqmode == kQGlobal) ? 2 : 1;
}

cudaError_t launch_decode(int codec, int rowbytes, int qmode, DecodeArgs a, cudaStream_t stream, bool after_append) {
  Plan pl;
  if (!plan_decode(codec, rowbytes, qmode, a, &pl)) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  void* args[] = {&a};
  if (pl.cluster) {
    cudaError_t e = ensure_smem(pl.ki.cfn, pl.smem);
    if (e != cudaSuccess) return e;
    a.ctas = pl.csize;
    a.dep = after_append ? 2 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.csize, a.H, a.B);
    cfg.blockDim = dim3(kDecodeThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = pl.csize;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = after_append ? attr : attr + 1;
    cfg.numAttrs = after_append ? 2 : 1;
    return cudaLaunchKernelExC(&cfg, pl.ki.cfn, args);
  }
  cudaError_t e = ensure_smem(pl.ki.fn, pl.smem);
  if (e != cudaSuccess) return e;
  a.ctas = pl.ctas;
  bool pdl = after_append;
  if (pl.ki.pqmode == kQGlobal) {
    // q' for every (b, h) first; the decode is launched behind it so that its
    // split plan and first tiles overlap the projection (only its helper warp
    // waits for q').  Behind an append the projection itself completes after
    // the append, and the decode waits for everything (dep 2).
    e = launch_qproj(a.B, a.H, a.Hd, a.W, a.q, a.q_dtype, a.Bk, a.sBk, a.w8, a.qglobal, stream, after_append);
    if (e != cudaSuccess) return e;
    a.dep = after_append ? 2 : 1;
    pdl = true;
  } else {
    a.dep = after_append ? 2 : 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.ctas);
  cfg.blockDim = dim3(kPersistThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, pl.ki.fn, args);
}

bool step_fused_applies(const AppendArgs& ap, const DecodeArgs& a) {
  StepPlan sp;
  return plan_step(ap, a, &sp);
}

cudaError_t launch_step_fused(const AppendArgs& ap, const DecodeArgs& a, cudaStream_t stream, bool* launched) {
  *launched = false;
  StepPlan sp;
  if (!plan_step(ap, a, &sp)) return cudaSuccess;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(sp.si.fn), sp.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sp.csize, a.H, 1);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = sp.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = sp.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ap.dep ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, sp.si.fn, a, ap);
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace wsvd
