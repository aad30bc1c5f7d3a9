// Building blocks of the latent append (rotation of the new token's x slice,
// the A row stream through a per-thread cp.async ring, the GEMV partials,
// their reduction across a CTA, and the quantiser of one finished row),
// shared by the append kernel and the one-kernel decode step so that both
// compute the appended rows with the same operations in the same order.
// All run on 256 threads (the consumer threads of the step kernel); `sync`
// is the barrier over those threads.
#pragma once

#include "common.cuh"

namespace wsvd {

constexpr int kAppendThreads = 256;
constexpr int kAppendWarps = kAppendThreads / 32;
constexpr int kRing = 8;  // A rows in flight per thread

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_ring() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 1) : "memory");
}

__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

// Per-thread share of the CTA's A slice: rows k * nrg + rg (k = 0, 1, ...) of
// the slice, 8 columns starting at 8 * cgi: one 16-byte piece per row (fp16),
// or 8 bytes (int8 A) in the first half of the ring slot.
template <bool W8>
struct RowWalk {
  const uint8_t* A;  // first row of the slice
  int r, Ec, nrg, rg, cgi, nrows;
  __device__ __forceinline__ bool valid(int k) const { return k < nrows; }
  __device__ __forceinline__ int row(int k) const { return k * nrg + rg; }
  __device__ __forceinline__ void issue(uint4* ring, int k, int tid) const {
    if (valid(k)) {
      const uint8_t* src = A + ((size_t)row(k) * r + cgi * 8) * (W8 ? 1 : 2);
      if (W8) cp_async8(ring + (size_t)(k % kRing) * kAppendThreads + tid, src);
      else cp_async16(ring + (size_t)(k % kRing) * kAppendThreads + tid, src);
    }
    cp_async_commit();  // one group per ring step, empty past the end
  }
};

// c[bb0 + bi][8 * cgi .. + 8] += xs[bb0 + bi][e] * A[e][8 * cgi .. + 8] for one
// A row piece av (8 fp16 values, or 8 int8 codes in av.x, av.y); acc[bi][k]
// holds columns 2k, 2k + 1 (packed fp32 FMAs, each lane rounded as fmaf).
template <int BB, bool W8>
__device__ __forceinline__ void accumulate_row(const uint4& av, const float* xs, int B, int bb0, int Ec, int e,
                                               float2 (&acc)[BB][4]) {
  float2 a[4];
  if (W8) {  // int8 codes -> fp32, exact
    a[0] = i8_pair(av.x ^ 0x80808080u, 0);
    a[1] = i8_pair(av.x ^ 0x80808080u, 2);
    a[2] = i8_pair(av.y ^ 0x80808080u, 0);
    a[3] = i8_pair(av.y ^ 0x80808080u, 2);
  } else {
    a[0] = h2_pair(av.x);
    a[1] = h2_pair(av.y);
    a[2] = h2_pair(av.z);
    a[3] = h2_pair(av.w);
  }
#pragma unroll
  for (int bi = 0; bi < BB; ++bi) {
    const float xv = (bb0 + bi < B) ? xs[(size_t)(bb0 + bi) * Ec + e] : 0.f;
    const float2 x2 = make_float2(xv, xv);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[bi][k] = __ffma2_rn(x2, a[k], acc[bi][k]);
  }
}

// Accumulate c[bb0 + bi][8 * cgi .. + 8] over this thread's rows, streaming
// them through the ring (rows 0 .. kRing-1 already issued by the caller).
template <int BB, bool W8>
__device__ __forceinline__ void stream_rows(const RowWalk<W8>& w, uint4* ring, const float* xs, int B, int bb0,
                                            float2 (&acc)[BB][4], int tid) {
#pragma unroll
  for (int bi = 0; bi < BB; ++bi)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[bi][k] = make_float2(0.f, 0.f);
  for (int k = 0; k < w.nrows; ++k) {
    cp_async_wait_ring();  // this thread's group k is complete
    const uint4 av = ring[(size_t)(k % kRing) * kAppendThreads + tid];
    // The slot is consumed (values in registers) before it is refilled.
    w.issue(ring, k + kRing, tid);
    accumulate_row<BB, W8>(av, xs, B, bb0, w.Ec, w.row(k), acc);
  }
}

// Pairwise sums over the lanes that share a column group (lane % NCG), in
// the order of a butterfly with partner lane ^ O for O = NCG, 2 NCG, ..., 16,
// halving the values every round while more than one is left: each sum is
// the one the full butterfly gives, bit for bit, with far fewer shuffles.
// Returns the index of this lane's first value; it keeps NV >> rounds values
// (at least one; lanes that differ only in the later rounds' bits then hold
// the same sum).
template <int NV, int O>
__device__ __forceinline__ int reduce_scatter_lanes(float* v, int lane) {
  if constexpr (O >= 32) {
    return 0;
  } else if constexpr (NV >= 2) {
    constexpr int HALF = NV / 2;
    const bool up = (lane & O) != 0;
#pragma unroll
    for (int j = 0; j < HALF; ++j) {
      const float send = up ? v[j] : v[j + HALF];
      const float keep = up ? v[j + HALF] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    return (up ? HALF : 0) + reduce_scatter_lanes<HALF, O * 2>(v, lane);
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
    return reduce_scatter_lanes<1, O * 2>(v, lane);
  }
}

// Reduce acc over the CTA (threads sharing a column group, then warps) into
// the slot rows bi < nb: a local store on the leader (remote_bar == 0), else an
// st.async into the leader's slot at cluster address remote_dst that completes
// 4 bytes per value on the leader's barrier.  Fixed summation order: within a
// warp the butterfly over the lanes of a column group (partners at offsets
// NCG, 2 NCG, ..., 16), then the warps in order.  NCG = r / 8 divides 32.
template <int BB, int NCG, typename Sync>
__device__ __forceinline__ void reduce_cta(float2 (&acc)[BB][4], int r, int nb, float* red, float* dst,
                                             uint32_t remote_dst, uint32_t remote_bar, int tid, Sync sync) {
  constexpr int NV = BB * 8;
  constexpr int ROUNDS = NCG == 1 ? 5 : NCG == 2 ? 4 : NCG == 4 ? 3 : NCG == 8 ? 2 : 1;
  constexpr int KEPT = (NV >> ROUNDS) > 0 ? (NV >> ROUNDS) : 1;
  const int warp = tid >> 5, lane = tid & 31, cgi = lane % NCG;
  float v[NV];
#pragma unroll
  for (int bi = 0; bi < BB; ++bi)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[bi * 8 + 2 * k] = acc[bi][k].x;
      v[bi * 8 + 2 * k + 1] = acc[bi][k].y;
    }
  const int base = reduce_scatter_lanes<NV, NCG>(v, lane);
#pragma unroll
  for (int i = 0; i < KEPT; ++i) {
    const int idx = base + i, bi = idx >> 3, k = idx & 7;
    red[(warp * BB + bi) * r + cgi * 8 + k] = v[i];
  }
  sync();
  for (int idx = tid; idx < nb * r; idx += kAppendThreads) {
    const int bi = idx / r, j = idx % r;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kAppendWarps; ++w) s += red[(w * BB + bi) * r + j];
    if (remote_bar) st_async_f32(remote_dst + 4u * (uint32_t)(bi * r + j), s, remote_bar);
    else dst[(size_t)bi * r + j] = s;
  }
  sync();
}


__device__ __forceinline__ float x_elem(uint32_t bits16, int dtype) {
  return dtype == WSVD_DTYPE_BF16 ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((uint16_t)bits16));
}

// Butterfly stage pairs (i, i + hh) of one Hadamard block held in shared memory.
__device__ __forceinline__ void fwht_smem_warp(float* v, int blk, int lane) {
  for (int hh = 1; hh < blk; hh <<= 1) {
    for (int q = lane; q < blk / 2; q += 32) {
      const int i = (q / hh) * 2 * hh + (q % hh);
      const float u = v[i], w = v[i + hh];
      v[i] = u + w;
      v[i + hh] = u - w;
    }
    __syncwarp();
  }
}


// x slice [e0, e0 + Ec) of every batch row: the registers of the fast path
// (128-element chunks per warp, lane holds 4 consecutive values), loaded
// through L2.
constexpr int kXChunks = 4;  // 128-element x chunks per warp held in registers (fast path)
__host__ __device__ inline bool x_fast_path(int B, int Ec, int blk) {
  return (Ec % 128 == 0) && blk <= 128 && B * Ec / 128 <= kXChunks * kAppendWarps;
}
__device__ __forceinline__ void load_x_slice(uint2 (&xraw)[kXChunks], const void* x, int B, int E, int e0, int Ec,
                                             int warp, int lane) {
  const int nch = B * Ec / 128;
  const uint16_t* xg = static_cast<const uint16_t*>(x);
#pragma unroll
  for (int t = 0; t < kXChunks; ++t) {
    const int ch = warp + t * kAppendWarps;
    if (ch < nch) {
      const int b = ch / (Ec / 128), off = (ch % (Ec / 128)) * 128;
      xraw[t] = __ldcg(reinterpret_cast<const uint2*>(xg + (size_t)b * E + e0 + off) + lane);
    }
  }
}

// Rotate the x slice into xs[b][e] (unnormalised: 1/sqrt(blk) is applied to
// c): in registers and warp shuffles when `fast` (xraw loaded), else through
// shared memory from global x.  Ends with `sync`.
template <typename Sync>
__device__ __forceinline__ void rotate_x_slice(bool fast, const uint2 (&xraw)[kXChunks], float* xs, const void* x,
                                               int x_dtype, int B, int E, int e0, int Ec, int blk, int tid, Sync sync) {
  const int warp = tid >> 5, lane = tid & 31;
  if (fast) {
    const int nch = B * Ec / 128;
    // lane holds elements 4*lane .. 4*lane+3 of a 128-element chunk
#pragma unroll
    for (int t = 0; t < kXChunks; ++t) {
      const int ch = warp + t * kAppendWarps;
      if (ch >= nch) continue;  // warp-uniform
      float v[4] = {x_elem(xraw[t].x & 0xffffu, x_dtype), x_elem(xraw[t].x >> 16, x_dtype),
                    x_elem(xraw[t].y & 0xffffu, x_dtype), x_elem(xraw[t].y >> 16, x_dtype)};
      if (blk >= 2) {
        const float u0 = v[0] + v[1], u1 = v[0] - v[1], u2 = v[2] + v[3], u3 = v[2] - v[3];
        v[0] = u0; v[1] = u1; v[2] = u2; v[3] = u3;
      }
      if (blk >= 4) {
        const float u0 = v[0] + v[2], u2 = v[0] - v[2], u1 = v[1] + v[3], u3 = v[1] - v[3];
        v[0] = u0; v[1] = u1; v[2] = u2; v[3] = u3;
      }
      for (int m = 1; 4 * m < blk; m <<= 1) {  // pair distance 4m = lane distance m
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float o = __shfl_xor_sync(0xffffffffu, v[k], m);
          v[k] = upper ? o - v[k] : v[k] + o;
        }
      }
      const int b = ch / (Ec / 128), off = (ch % (Ec / 128)) * 128;
      *reinterpret_cast<float4*>(xs + (size_t)b * Ec + off + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
    }
  } else {
    const uint16_t* xg = static_cast<const uint16_t*>(x);
    for (int i = tid; i < B * Ec; i += kAppendThreads) {
      const int b = i / Ec, e = i % Ec;
      xs[i] = x_elem(xg[(size_t)b * E + e0 + e], x_dtype);
    }
    sync();
    const int nblk = B * (Ec / blk);
    for (int bk = warp; bk < nblk; bk += kAppendWarps) fwht_smem_warp(xs + (size_t)bk * blk, blk, lane);
  }
  sync();
}

// The int8 weights' column scales of the columns a lane quantises (j = lane +
// 32 k), loaded ahead of the quantiser so that their latency is hidden.
template <int RMAX>
struct ColScales {
  static constexpr int K = (RMAX + 31) / 32;
  float v[K];
  __device__ __forceinline__ void load(const float* colscale, int r, int lane) {
#pragma unroll
    for (int k = 0; k < K; ++k) v[k] = (lane + 32 * k < r) ? __ldg(colscale + lane + 32 * k) : 1.f;
  }
};

// Quantise one finished row of one (b, h, K|V) unit, one warp: the cluster
// ranks' partial sums (slots[q * stride + j], q = 0 .. nranks - 1) added in
// rank order, times 1/sqrt(blk) (and the int8 weights' column scale, from cs),
// then the append's fp32 decisions; the codes are written to dst when `ok`
// (and to dst2 too, when given).  Returns the fp16 scale.  RMAX: a bound on r
// known at compile time (128 covers every r; a caller with a fixed r passes it).
template <bool W8, int RMAX = 128>
__device__ __forceinline__ __half quantise_append_row(const float* slots, size_t stride, int nranks, int r, int bits,
                                                      float hnorm, const ColScales<RMAX>& cs, bool ok, uint8_t* dst,
                                                      uint8_t* dst2, int lane) {
  constexpr int KMAX = (RMAX + 31) / 32;  // column groups of 32 a lane may hold
  const int Q = (bits == 8) ? 127 : 7;
  float cv[KMAX];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    const int j = lane + 32 * k;
    cv[k] = 0.f;
    if (j < r) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q)  // clusters hold at most 8 ranks
        if (q < nranks) sum += slots[(size_t)q * stride + j];
      cv[k] = sum * hnorm;
      if (W8) cv[k] *= cs.v[k];  // column scale of int8 A
      amax = fmaxf(amax, fabsf(cv[k]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half sh = __float2half_rn(__fdiv_rn(amax, (float)Q));
  const float sc = __half2float(sh);
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    if (32 * k >= r) break;  // no column of this group (uniform across the warp)
    const int j = lane + 32 * k;
    const int code = sc > 0.f ? max(-Q, min(Q, __float2int_rn(__fdiv_rn(cv[k], sc)))) : 0;
    if (bits == 8) {
      if (ok && j < r) {
        dst[j] = (uint8_t)code;
        if (dst2) dst2[j] = (uint8_t)code;
      }
    } else {
      const int hi = __shfl_down_sync(0xffffffffu, code, 1);  // column j + 1 (r is a multiple of 8)
      if (ok && j < r && (lane & 1) == 0) {
        const uint8_t v = (uint8_t)((code & 0xF) | ((hi & 0xF) << 4));
        dst[j / 2] = v;
        if (dst2) dst2[j / 2] = v;
      }
    }
  }
  return sh;
}

}  // namespace wsvd
