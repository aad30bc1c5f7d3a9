// Persistent split-L flash-decoding over a low-rank (int8 / int4) or dense
// (fp16) cache, for sm_100a.
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
// Work decomposition: the (b, h, tile) space of all sequences is flattened
// (tiles of T tokens, t fastest) and split evenly over a persistent grid of C
// CTAs, so ragged lengths cost nothing extra.  A CTA that crosses a (b, h)
// boundary writes one partial (m, l, o[W]) per (b, h) it touched, into slot
// c + b*H + h (slots of consecutive CTAs never collide because tile ranges are
// ordered).  combine_kernel merges the partials of each (b, h) and applies
// B_Vh.
//
// Per CTA: one producer warp issues 1-D bulk copies (TMA, no multicast) of
// K codes, V codes and their scales into a kStages-deep shared-memory ring;
// eight consumer warps read 16-byte segments (a token's row is split over
// SEGS adjacent lanes), convert codes to fp32 exactly, keep a per-thread
// online softmax and reduce across lanes / warps only at (b, h) boundaries.
#include "common.cuh"

namespace wsvd {

template <int CODEC>
struct CodecT;
template <>
struct CodecT<kCodecI8> {
  static constexpr int kVals = 16;  // values per 16-byte segment
  static constexpr bool kScaled = true;
};
template <>
struct CodecT<kCodecI4> {
  static constexpr int kVals = 32;
  static constexpr bool kScaled = true;
};
template <>
struct CodecT<kCodecF16> {
  static constexpr int kVals = 8;
  static constexpr bool kScaled = false;
};

// ------------------------------------------------------------------ segment math
// q2 / acc point at the thread's float2 pairs for this segment (kVals / 2 pairs).
template <int CODEC>
__device__ __forceinline__ void seg_dot(const uint4 s, const float2* q2, float2& d0, float2& d1);
template <int CODEC>
__device__ __forceinline__ void seg_axpy(const uint4 s, const float2 w, float2* acc);

template <>
__device__ __forceinline__ void seg_dot<kCodecI8>(const uint4 s, const float2* q2, float2& d0, float2& d1) {
  const uint32_t w[4] = {s.x ^ 0x80808080u, s.y ^ 0x80808080u, s.z ^ 0x80808080u, s.w ^ 0x80808080u};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    d0 = __ffma2_rn(i8_pair(w[k], 0), q2[2 * k], d0);
    d1 = __ffma2_rn(i8_pair(w[k], 2), q2[2 * k + 1], d1);
  }
}
template <>
__device__ __forceinline__ void seg_axpy<kCodecI8>(const uint4 s, const float2 w2, float2* acc) {
  const uint32_t w[4] = {s.x ^ 0x80808080u, s.y ^ 0x80808080u, s.z ^ 0x80808080u, s.w ^ 0x80808080u};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc[2 * k] = __ffma2_rn(i8_pair(w[k], 0), w2, acc[2 * k]);
    acc[2 * k + 1] = __ffma2_rn(i8_pair(w[k], 2), w2, acc[2 * k + 1]);
  }
}

template <>
__device__ __forceinline__ void seg_dot<kCodecI4>(const uint4 s, const float2* q2, float2& d0, float2& d1) {
  const uint32_t w[4] = {s.x ^ 0x88888888u, s.y ^ 0x88888888u, s.z ^ 0x88888888u, s.w ^ 0x88888888u};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    d0 = __ffma2_rn(i4_pair(w[k], 0), q2[4 * k + 0], d0);
    d1 = __ffma2_rn(i4_pair(w[k], 2), q2[4 * k + 1], d1);
    d0 = __ffma2_rn(i4_pair(w[k], 4), q2[4 * k + 2], d0);
    d1 = __ffma2_rn(i4_pair(w[k], 6), q2[4 * k + 3], d1);
  }
}
template <>
__device__ __forceinline__ void seg_axpy<kCodecI4>(const uint4 s, const float2 w2, float2* acc) {
  const uint32_t w[4] = {s.x ^ 0x88888888u, s.y ^ 0x88888888u, s.z ^ 0x88888888u, s.w ^ 0x88888888u};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[4 * k + p] = __ffma2_rn(i4_pair(w[k], 2 * p), w2, acc[4 * k + p]);
  }
}

template <>
__device__ __forceinline__ void seg_dot<kCodecF16>(const uint4 s, const float2* q2, float2& d0, float2& d1) {
  d0 = __ffma2_rn(h2_pair(s.x), q2[0], d0);
  d1 = __ffma2_rn(h2_pair(s.y), q2[1], d1);
  d0 = __ffma2_rn(h2_pair(s.z), q2[2], d0);
  d1 = __ffma2_rn(h2_pair(s.w), q2[3], d1);
}
template <>
__device__ __forceinline__ void seg_axpy<kCodecF16>(const uint4 s, const float2 w2, float2* acc) {
  acc[0] = __ffma2_rn(h2_pair(s.x), w2, acc[0]);
  acc[1] = __ffma2_rn(h2_pair(s.y), w2, acc[1]);
  acc[2] = __ffma2_rn(h2_pair(s.z), w2, acc[2]);
  acc[3] = __ffma2_rn(h2_pair(s.w), w2, acc[3]);
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

template <int CODEC, int SEGS, int SPT>
struct SplitCfg {
  using CT = CodecT<CODEC>;
  static constexpr int kVS = CT::kVals;
  static constexpr int kVals = kVS * SPT;            // values per consumer thread
  static constexpr int kPairs = kVals / 2;
  static constexpr int kT = kConsumerThreads / SEGS;  // tokens per tile
  static constexpr int kRB = SEGS * SPT * 16;         // bytes per token row
  static constexpr int kW = SEGS * SPT * kVS;         // values per token row
  static constexpr int kCodeBytes = kT * kRB;
  static constexpr int kScaleBytes = CT::kScaled ? kT * 2 : 0;
  static constexpr int kStageBytes = 2 * kCodeBytes + 2 * kScaleBytes;
  static constexpr int kRedFloats = kConsumerWarps * SEGS * (kVals + 2);
  static_assert(kT % 8 == 0, "tile must hold a multiple of 8 tokens (16-byte scale copies)");
  static size_t smem_bytes(int B) {
    return (size_t)kStages * kStageBytes + 2 * kStages * sizeof(uint64_t) + (size_t)kW * 4 +
           (size_t)kRedFloats * 4 + (size_t)(B + 1) * 4;
  }
};

template <int CODEC, int SEGS, int SPT, int QMODE>
__global__ void __launch_bounds__(kDecodeThreads, 2) split_decode_kernel(const SplitArgs a) {
  using C = SplitCfg<CODEC, SEGS, SPT>;
  using CT = typename C::CT;
  constexpr int VS = C::kVS, VALS = C::kVals, NP = C::kPairs, T = C::kT, RB = C::kRB, W = C::kW;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes);
  uint64_t* empty = full + kStages;
  float* qs = reinterpret_cast<float*>(empty + kStages);
  float* red = qs + W;
  int* pre = reinterpret_cast<int*>(red + C::kRedFloats);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;

  // Tiles per sequence (per head), exclusive prefix over sequences.
  if (warp == 0) {
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) {
      const int raw = a.seq_lens[b];
      if ((raw < 0 || raw > a.L_cap) && c == 0) set_err(a.err, WSVD_DEVERR_LEN_RANGE);
      sum += (clamp_len(raw, a.L_cap) + T - 1) / T;
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
      run += (clamp_len(a.seq_lens[b], a.L_cap) + T - 1) / T;
    }
    if (lane == 31) pre[a.B] = incl;
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], kConsumerWarps);
      }
      fence_mbar_init();
    }
  }
  __syncthreads();

  const TileWalk walk{pre, a.B, a.H};
  const long long G = (long long)a.H * pre[a.B];
  const long long g_begin = G * c / a.ctas, g_end = G * (c + 1) / a.ctas;
  if (g_begin >= g_end) return;  // uniform across the CTA; nothing was issued

  // ---------------------------------------------------------------- producer warp
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      int b, h, t;
      walk.locate(g_begin, b, h, t);
      long long issued = 0;
      bool ok = true;
      for (long long g = g_begin; g < g_end; ++g, ++issued) {
        const int s = (int)(issued % kStages);
        if (issued >= kStages && !mbar_wait_bounded(&empty[s], (uint32_t)(((issued / kStages) - 1) & 1))) {
          set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
          ok = false;
          break;
        }
        const int len = a.seq_lens[b];
        const int n = min(T, len - t * T);
        const size_t head_row = ((size_t)b * a.H + h) * a.L_cap + (size_t)t * T;
        const size_t row0 = a.heads_share ? (size_t)b * a.L_cap + (size_t)t * T : head_row;
        uint8_t* st = stages + s * C::kStageBytes;
        const uint32_t cb = (uint32_t)n * RB;
        const uint32_t sb = CT::kScaled ? (uint32_t)((n + 7) & ~7) * 2u : 0u;
        mbar_arrive_expect_tx(&full[s], 2 * cb + 2 * sb);
        bulk_g2s(st, a.lat_k + row0 * RB, cb, &full[s], pol);
        bulk_g2s(st + C::kCodeBytes, a.lat_v + row0 * RB, cb, &full[s], pol);
        if (CT::kScaled) {
          bulk_g2s(st + 2 * C::kCodeBytes, a.scale_k + head_row, sb, &full[s], pol);
          bulk_g2s(st + 2 * C::kCodeBytes + C::kScaleBytes, a.scale_v + head_row, sb, &full[s], pol);
        }
        walk.advance(b, h, t);
      }
      // Leave no copy in flight behind: wait (bounded) for the last uses of each stage.
      const long long last = issued;
      for (long long i = (last > kStages ? last - kStages : 0); i < last && ok; ++i) {
        const int s = (int)(i % kStages);
        if (!mbar_wait_bounded(&full[s], (uint32_t)((i / kStages) & 1))) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumer warps
  const int tok = tid / SEGS, sl = tid % SEGS;
  float2 qv[NP], acc[NP];
  float m = kNegInf, l = 0.f;
  bool timed_out = false;

  auto setup_query = [&](int b, int h) {
    if (QMODE == kQProj) {
      // q' = B_Kh . q, scaled by softmax_scale * log2(e): one warp per row of B_Kh.
      const size_t qoff = ((size_t)b * a.H + h) * a.Hd;
      float qr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        qr[k] = (lane + 32 * k < a.Hd) ? load_q_elem(a.q, a.q_dtype, qoff + lane + 32 * k) : 0.f;
      const __half* Bh = a.Bk + (size_t)h * W * a.Hd;
      for (int j = warp; j < W; j += kConsumerWarps) {
        float d = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (lane + 32 * k < a.Hd) d = fmaf(__half2float(Bh[(size_t)j * a.Hd + lane + 32 * k]), qr[k], d);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) qs[j] = d * a.qscale;
      }
    } else if (QMODE == kQDirect) {
      const size_t qoff = ((size_t)b * a.H + h) * a.Hd;
      for (int j = tid; j < W; j += kConsumerThreads) qs[j] = load_q_elem(a.q, a.q_dtype, qoff + j) * a.qscale;
    } else {
      const float* qg = a.qglobal + ((size_t)b * a.H + h) * W;
      for (int j = tid; j < W; j += kConsumerThreads) qs[j] = qg[j] * a.qscale;
    }
    named_barrier_sync(1, kConsumerThreads);
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
      const int e0 = (sl + i * SEGS) * VS;
#pragma unroll
      for (int p = 0; p < VS / 2; ++p) qv[i * (VS / 2) + p] = make_float2(qs[e0 + 2 * p], qs[e0 + 2 * p + 1]);
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) acc[p] = make_float2(0.f, 0.f);
    m = kNegInf;
    l = 0.f;
  };

  auto flush = [&](int b, int h) {
    // Merge lanes that hold the same segment (same sl), then warps.
#pragma unroll
    for (int o = SEGS; o < 32; o <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m, o);
      const float lo = __shfl_xor_sync(0xffffffffu, l, o);
      const float M = fmaxf(m, mo);
      const float f1 = (m == kNegInf) ? 0.f : exp2f(m - M);
      const float f2 = (mo == kNegInf) ? 0.f : exp2f(mo - M);
      l = l * f1 + lo * f2;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        float2 ao;
        ao.x = __shfl_xor_sync(0xffffffffu, acc[p].x, o);
        ao.y = __shfl_xor_sync(0xffffffffu, acc[p].y, o);
        acc[p] = __ffma2_rn(acc[p], make_float2(f1, f1), __fmul2_rn(ao, make_float2(f2, f2)));
      }
      m = M;
    }
    if (lane < SEGS) {
      float* rw = red + (warp * SEGS + sl) * (VALS + 2);
      rw[0] = m;
      rw[1] = l;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        rw[2 + 2 * p] = acc[p].x;
        rw[3 + 2 * p] = acc[p].y;
      }
    }
    named_barrier_sync(1, kConsumerThreads);
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[w * SEGS * (VALS + 2)]);
    float f[kConsumerWarps];
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = red[w * SEGS * (VALS + 2)];
      f[w] = (mw == kNegInf) ? 0.f : exp2f(mw - M);
    }
    float* dst = a.partials + ((size_t)c + (size_t)b * a.H + h) * (W + 2);
    for (int e = tid; e < W; e += kConsumerThreads) {
      const int seg = e / VS, sle = seg % SEGS, v = (seg / SEGS) * VS + e % VS;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) s = fmaf(f[w], red[(w * SEGS + sle) * (VALS + 2) + 2 + v], s);
      dst[2 + e] = s;
    }
    if (tid == 0) {
      float ls = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) ls = fmaf(f[w], red[w * SEGS * (VALS + 2) + 1], ls);
      dst[0] = M;
      dst[1] = ls;
    }
    named_barrier_sync(1, kConsumerThreads);
  };

  int b, h, t;
  walk.locate(g_begin, b, h, t);
  int cb = -1, ch = -1;
  long long i = 0;
  for (long long g = g_begin; g < g_end; ++g, ++i) {
    if (b != cb || h != ch) {
      if (cb >= 0) flush(cb, ch);
      setup_query(b, h);
      cb = b;
      ch = h;
    }
    const int s = (int)(i % kStages);
    // A timed-out wait only poisons the result (err is set); control flow stays
    // uniform so every consumer warp reaches every named barrier.
    if (!mbar_wait_bounded(&full[s], (uint32_t)((i / kStages) & 1), timed_out ? 0ull : kWaitLimitNs)) {
      if (!timed_out && lane == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
      timed_out = true;
    }
    const int n = min(T, a.seq_lens[b] - t * T);
    const bool valid = tok < n;
    const uint8_t* st = stages + s * C::kStageBytes;
    const uint8_t* rowk = st + tok * RB;
    const uint8_t* rowv = st + C::kCodeBytes + tok * RB;

    float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < SPT; ++j) {
      const uint4 kc = *reinterpret_cast<const uint4*>(rowk + (sl + j * SEGS) * 16);
      seg_dot<CODEC>(kc, &qv[j * (VS / 2)], d0, d1);
    }
    float d = (d0.x + d0.y) + (d1.x + d1.y);
#pragma unroll
    for (int o = 1; o < SEGS; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);

    float sk = 1.f, sv = 1.f;
    if (CT::kScaled && valid) {
      const __half* scl = reinterpret_cast<const __half*>(st + 2 * C::kCodeBytes);
      sk = __half2float(scl[tok]);
      sv = __half2float(scl[T + tok]);
    }
    const float sc = valid ? d * sk : kNegInf;
    if (sc > m + 8.f) {  // lazy rescale: the reference max moves only when a score beats it by 2^8
      const float fr = exp2f(m - sc);
      l *= fr;
#pragma unroll
      for (int p = 0; p < NP; ++p) acc[p] = __fmul2_rn(acc[p], make_float2(fr, fr));
      m = sc;
    }
    if (valid) {
      const float p = exp2f(sc - m);
      l += p;
      const float wv = p * sv;
#pragma unroll
      for (int j = 0; j < SPT; ++j) {
        const uint4 vc = *reinterpret_cast<const uint4*>(rowv + (sl + j * SEGS) * 16);
        seg_axpy<CODEC>(vc, make_float2(wv, wv), &acc[j * (VS / 2)]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    walk.advance(b, h, t);
  }
  if (cb >= 0) flush(cb, ch);
}

// ------------------------------------------------------------------ combine
// One CTA per (b, h): merge the partials of every CTA that touched (b, h),
// then up-project through B_Vh (low-rank paths) or normalise (dense path).
__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
  __shared__ float f[kMaxDecodeCtas];
  __shared__ int red_i[2][8];
  __shared__ float red_f[8];
  extern __shared__ float o[];  // W floats

  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.tile;

  // Tiles of sequences < b and of all sequences.
  int before = 0, total = 0;
  for (int i = tid; i < a.B; i += blockDim.x) {
    const int tb = (clamp_len(a.seq_lens[i], a.L_cap) + T - 1) / T;
    total += tb;
    if (i < b) before += tb;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, off);
    total += __shfl_xor_sync(0xffffffffu, total, off);
  }
  if (lane == 0) {
    red_i[0][warp] = before;
    red_i[1][warp] = total;
  }
  __syncthreads();
  before = total = 0;
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
    before += red_i[0][w];
    total += red_i[1][w];
  }
  const int len = clamp_len(a.seq_lens[b], a.L_cap);
  const int tb = (len + T - 1) / T;
  float* outp = a.out + (size_t)bh * a.Hd;
  if (tb == 0) {
    for (int d = tid; d < a.Hd; d += blockDim.x) outp[d] = 0.f;
    return;
  }
  const long long G = (long long)a.H * total;
  const long long g0 = (long long)a.H * before + (long long)h * tb, g1 = g0 + tb - 1;
  auto cta_of = [&](long long g) { return (int)(((g + 1) * a.ctas + G - 1) / G - 1); };
  const int c0 = cta_of(g0), c1 = cta_of(g1);
  const int np = c1 - c0 + 1;
  const int W = a.W;
  const float* part = a.partials + ((size_t)c0 + bh) * (W + 2);

  float M = kNegInf;
  for (int p = tid; p < np; p += blockDim.x) M = fmaxf(M, part[(size_t)p * (W + 2)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) red_f[warp] = M;
  __syncthreads();
  M = kNegInf;
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) M = fmaxf(M, red_f[w]);
  for (int p = tid; p < np; p += blockDim.x) {
    const float mp = part[(size_t)p * (W + 2)];
    f[p] = (mp == kNegInf) ? 0.f : exp2f(mp - M);
  }
  __syncthreads();
  float lsum = 0.f;
  for (int p = 0; p < np; ++p) lsum = fmaf(f[p], part[(size_t)p * (W + 2) + 1], lsum);
  for (int e = tid; e < W; e += blockDim.x) {
    float s = 0.f;
    for (int p = 0; p < np; ++p) s = fmaf(f[p], part[(size_t)p * (W + 2) + 2 + e], s);
    o[e] = s;
  }
  __syncthreads();
  const float inv = 1.f / lsum;
  if (a.Bv == nullptr) {
    for (int d = tid; d < a.Hd; d += blockDim.x) outp[d] = o[d] * inv;
  } else {
    const __half* Bh = a.Bv + (size_t)h * W * a.Hd;
    for (int d = tid; d < a.Hd; d += blockDim.x) {
      float s = 0.f;
      for (int e = 0; e < W; ++e) s = fmaf(o[e], __half2float(Bh[(size_t)e * a.Hd + d]), s);
      outp[d] = s * inv;
    }
  }
}

// ------------------------------------------------------------------ host side
namespace {

struct KernelInfo {
  const void* fn;
  size_t smem_fixed;  // bytes without the (B + 1) prefix ints
  int tile;
};

template <int CODEC, int SEGS, int SPT, int QMODE>
KernelInfo info() {
  using C = SplitCfg<CODEC, SEGS, SPT>;
  return KernelInfo{reinterpret_cast<const void*>(&split_decode_kernel<CODEC, SEGS, SPT, QMODE>),
                    C::smem_bytes(0) - 4, C::kT};
}

// Supported instantiations: rows of 16..128 bytes for the quantised codecs,
// 64..512 bytes (fp16 Hd 32..256) for dense, 256..2048 bytes for shared latents.
bool pick(int codec, int rowbytes, int qmode, KernelInfo* ki) {
  const int nseg = rowbytes / 16;
  if (rowbytes % 16 || nseg < 1) return false;
  if (qmode == kQProj && codec == kCodecI8) {
    switch (nseg) {
      case 1: *ki = info<kCodecI8, 1, 1, kQProj>(); return true;
      case 2: *ki = info<kCodecI8, 2, 1, kQProj>(); return true;
      case 4: *ki = info<kCodecI8, 4, 1, kQProj>(); return true;
      case 8: *ki = info<kCodecI8, 8, 1, kQProj>(); return true;
    }
  } else if (qmode == kQProj && codec == kCodecI4) {
    switch (nseg) {
      case 1: *ki = info<kCodecI4, 1, 1, kQProj>(); return true;
      case 2: *ki = info<kCodecI4, 2, 1, kQProj>(); return true;
      case 4: *ki = info<kCodecI4, 4, 1, kQProj>(); return true;
      case 8: *ki = info<kCodecI4, 8, 1, kQProj>(); return true;
    }
  } else if (qmode == kQDirect && codec == kCodecF16) {
    switch (nseg) {
      case 8: *ki = info<kCodecF16, 8, 1, kQDirect>(); return true;
      case 16: *ki = info<kCodecF16, 16, 1, kQDirect>(); return true;
      case 32: *ki = info<kCodecF16, 32, 1, kQDirect>(); return true;
    }
  } else if (qmode == kQGlobal && codec == kCodecF16) {
    switch (nseg) {
      case 16: *ki = info<kCodecF16, 16, 1, kQGlobal>(); return true;
      case 32: *ki = info<kCodecF16, 32, 1, kQGlobal>(); return true;
      case 64: *ki = info<kCodecF16, 32, 2, kQGlobal>(); return true;
      case 128: *ki = info<kCodecF16, 32, 4, kQGlobal>(); return true;
    }
  }
  return false;
}

}  // namespace

int split_decode_tile_tokens(int codec, int rowbytes) {
  KernelInfo ki;
  for (int qm : {kQProj, kQDirect, kQGlobal})
    if (pick(codec, rowbytes, qm, &ki)) return ki.tile;
  return 0;
}

int split_decode_grid(int codec, int rowbytes, int qmode, int B, int H, int L_cap) {
  KernelInfo ki;
  if (!pick(codec, rowbytes, qmode, &ki)) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = ki.smem_fixed + (size_t)(B + 1) * 4;
  int occ = 1;
  cudaFuncSetAttribute(ki.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ki.fn, kDecodeThreads, smem) != cudaSuccess || occ < 1)
    occ = 1;
  const long long tiles_max = (long long)B * H * ((L_cap + ki.tile - 1) / ki.tile);
  long long ctas = (long long)sms * occ;
  if (ctas > tiles_max) ctas = tiles_max;
  if (ctas > kMaxDecodeCtas) ctas = kMaxDecodeCtas;
  if (ctas < 1) ctas = 1;
  return (int)ctas;
}

cudaError_t launch_split_decode(int codec, int rowbytes, int qmode, const SplitArgs& a, int* tile_tokens,
                                cudaStream_t stream) {
  KernelInfo ki;
  if (!pick(codec, rowbytes, qmode, &ki)) return cudaErrorInvalidValue;
  if (tile_tokens) *tile_tokens = ki.tile;
  const size_t smem = ki.smem_fixed + (size_t)(a.B + 1) * 4;
  cudaError_t e = cudaFuncSetAttribute(ki.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* args[] = {const_cast<SplitArgs*>(&a)};
  return cudaLaunchKernel(ki.fn, dim3(a.ctas), dim3(kDecodeThreads), args, smem, stream);
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  const size_t smem = (size_t)a.W * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  combine_kernel<<<a.B * a.H, 256, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace wsvd
