// Latent append for sm_100a: rotate the new token's activation with the block
// Hadamard S1, project it through A_Kh / A_Vh and quantise each (b, h, K|V)
// row into the cache (WSVD summaries: German §2.A for the per-head projection
// W_Kh ~= A_Kh . B_Kh, German §2.C for the Hadamard rotation S1 and the
// W8A8 / W8A4 quantisation).
//
// The work is a GEMV [B x E] . [E x r] per (h, K|V) unit, bound by reading A
// (2 * H * E * r fp16).  Each unit is split over a thread-block cluster of
// up to 8 CTAs along E; every CTA pulls its contiguous A slice with one 1-D
// bulk copy (TMA, no multicast), rotates its slice of x with an in-place fast
// Walsh-Hadamard transform in shared memory, and reduces its slice to a
// partial c[B][r].  The cluster's leader sums the partials through
// distributed shared memory in a fixed order (deterministic), quantises and
// writes the row.  The last leader to finish (a completion counter in the
// caller's workspace, reset to zero by that leader) advances seq_lens.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace wsvd {

constexpr int kAppendThreads = 256;
constexpr int kAppendBB = 4;  // batches per pass over the A slice

struct AppendSmem {
  size_t a_off, x_off, part_off, red_off, cfin_off, codes_off, bar_off, total;
};

static __host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static __host__ __device__ inline AppendSmem append_layout(int B, int Ec, int r) {
  AppendSmem s;
  size_t o = 0;
  s.a_off = o;
  o = align_up(o + (size_t)Ec * r * 2, 16);
  s.x_off = o;
  o = align_up(o + (size_t)B * Ec * 4, 16);
  s.part_off = o;
  o = align_up(o + (size_t)B * r * 4, 16);
  s.red_off = o;
  o = align_up(o + (size_t)(kAppendThreads / 32) * kAppendBB * r * 4, 16);
  s.cfin_off = o;
  o = align_up(o + (size_t)B * r * 4, 16);
  s.codes_off = o;
  o = align_up(o + (size_t)B * r, 16);
  s.bar_off = o;
  o += 16;
  s.total = o;
  return s;
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.y, h = unit >> 1, kv = unit & 1;
  const int B = a.B, r = a.r, E = a.E;
  const int Ec = E / a.cluster, e0 = rank * Ec;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const AppendSmem L = append_layout(B, Ec, r);

  extern __shared__ __align__(128) uint8_t smem[];
  const __half* As = reinterpret_cast<const __half*>(smem + L.a_off);
  float* xs = reinterpret_cast<float*>(smem + L.x_off);
  float* part = reinterpret_cast<float*>(smem + L.part_off);
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  float* cfin = reinterpret_cast<float*>(smem + L.cfin_off);
  int8_t* codes = reinterpret_cast<int8_t*>(smem + L.codes_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar_off);

  // 1. Start the A slice on its way.
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    const uint8_t* src =
        reinterpret_cast<const uint8_t*>((kv ? a.Av : a.Ak) + ((size_t)h * E + e0) * (size_t)r);
    const uint32_t bytes = (uint32_t)Ec * r * 2;
    const uint64_t pol = l2_evict_first_policy();
    mbar_arrive_expect_tx(bar, bytes);
    constexpr uint32_t kPiece = 32768;
    for (uint32_t off = 0; off < bytes; off += kPiece)
      bulk_g2s(smem + L.a_off + off, src + off, min(kPiece, bytes - off), bar, pol);
  }

  // 2. x slice -> fp32, then the Walsh-Hadamard butterflies inside each block.
  for (int idx = tid; idx < B * Ec; idx += kAppendThreads) {
    const int b = idx / Ec, e = idx % Ec;
    xs[idx] = load_q_elem(a.x, a.x_dtype, (size_t)b * E + e0 + e);
  }
  __syncthreads();
  const int half_n = Ec / 2;
  for (int hh = 1; hh < a.blk; hh <<= 1) {
    for (int p = tid; p < B * half_n; p += kAppendThreads) {
      const int b = p / half_n, q = p % half_n;
      const int i = (q / hh) * 2 * hh + (q % hh);
      float* xb = xs + (size_t)b * Ec;
      const float u = xb[i], v = xb[i + hh];
      xb[i] = u + v;
      xb[i + hh] = u - v;
    }
    __syncthreads();
  }

  // 3. Wait for A (bounded), then the slice GEMV.
  if (!mbar_wait_bounded(bar, 0) && tid == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
  const int ncg = r / 8, nrg = kAppendThreads / ncg;
  const int cgi = tid % ncg, rg = tid / ncg;
  for (int bb0 = 0; bb0 < B; bb0 += kAppendBB) {
    float acc[kAppendBB][8];
#pragma unroll
    for (int bi = 0; bi < kAppendBB; ++bi)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[bi][k] = 0.f;
    for (int e = rg; e < Ec; e += nrg) {
      const uint4 av = *reinterpret_cast<const uint4*>(As + (size_t)e * r + cgi * 8);
      const float2 a01 = h2_pair(av.x), a23 = h2_pair(av.y), a45 = h2_pair(av.z), a67 = h2_pair(av.w);
      const float af[8] = {a01.x, a01.y, a23.x, a23.y, a45.x, a45.y, a67.x, a67.y};
#pragma unroll
      for (int bi = 0; bi < kAppendBB; ++bi) {
        if (bb0 + bi < B) {
          const float xv = xs[(size_t)(bb0 + bi) * Ec + e];
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[bi][k] = fmaf(xv, af[k], acc[bi][k]);
        }
      }
    }
    for (int o = ncg; o < 32; o <<= 1)
#pragma unroll
      for (int bi = 0; bi < kAppendBB; ++bi)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[bi][k] += __shfl_xor_sync(0xffffffffu, acc[bi][k], o);
    if (lane < ncg) {
#pragma unroll
      for (int bi = 0; bi < kAppendBB; ++bi)
#pragma unroll
        for (int k = 0; k < 8; ++k) red[(warp * kAppendBB + bi) * r + lane * 8 + k] = acc[bi][k];
    }
    __syncthreads();
    for (int idx = tid; idx < kAppendBB * r; idx += kAppendThreads) {
      const int bi = idx / r, j = idx % r;
      if (bb0 + bi < B) {
        float s = 0.f;
        for (int w = 0; w < kAppendThreads / 32; ++w) s += red[(w * kAppendBB + bi) * r + j];
        part[(size_t)(bb0 + bi) * r + j] = s;
      }
    }
    __syncthreads();
  }

  // 4. Cluster reduction and quantisation in the leader.
  cluster.sync();
  if (rank == 0) {
    for (int idx = tid; idx < B * r; idx += kAppendThreads) {
      float s = 0.f;
      for (int q = 0; q < a.cluster; ++q) s += cluster.map_shared_rank(part, q)[idx];
      cfin[idx] = s * a.hnorm;
    }
    __syncthreads();
    const int Q = (a.bits == 8) ? 127 : 7;
    const int RB = r * a.bits / 8;
    for (int b = warp; b < B; b += kAppendThreads / 32) {
      const int pos = a.seq_lens[b];
      const bool ok = pos >= 0 && pos < a.L_cap;
      const float* cb = cfin + (size_t)b * r;
      float amax = 0.f;
      for (int j = lane; j < r; j += 32) amax = fmaxf(amax, fabsf(cb[j]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const __half sh = __float2half_rn(__fdiv_rn(amax, (float)Q));
      const float s = __half2float(sh);
      for (int j = lane; j < r; j += 32) {
        int code = 0;
        if (s > 0.f) code = max(-Q, min(Q, __float2int_rn(__fdiv_rn(cb[j], s))));
        codes[b * r + j] = (int8_t)code;
      }
      __syncwarp();
      if (ok) {
        const size_t row = ((size_t)b * a.H + h) * a.L_cap + pos;
        uint32_t* dst = reinterpret_cast<uint32_t*>((kv ? a.lat_v : a.lat_k) + row * RB);
        for (int wi = lane; wi < RB / 4; wi += 32) {
          uint32_t word = 0;
          if (a.bits == 8) {
#pragma unroll
            for (int k = 0; k < 4; ++k) word |= (uint32_t)(uint8_t)codes[b * r + 4 * wi + k] << (8 * k);
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) word |= ((uint32_t)codes[b * r + 8 * wi + k] & 0xFu) << (4 * k);
          }
          dst[wi] = word;
        }
        if (lane == 0) (kv ? a.scale_v : a.scale_k)[row] = sh;
      } else if (lane == 0 && unit == 0) {
        set_err(a.err, WSVD_DEVERR_CACHE_FULL);
      }
    }
  }
  cluster.sync();  // every CTA's partial stays readable until the leader is done

  // 5. The last leader to finish advances the lengths.
  if (rank == 0 && tid == 0) {
    __threadfence();
    const int prev = atomicAdd(a.counter, 1);
    if (prev == (int)gridDim.y - 1) {
      __threadfence();
      for (int b = 0; b < B; ++b) {
        const int pos = a.seq_lens[b];
        if (pos >= 0 && pos < a.L_cap) a.seq_lens[b] = pos + 1;
      }
      atomicExch(a.counter, 0);
    }
  }
}

int append_cluster_size(int E, int blk) {
  for (int cl = 8; cl >= 1; cl >>= 1)
    if (E % (cl * blk) == 0) return cl;
  return 0;
}

size_t append_smem_bytes(int B, int E, int r, int cluster) { return append_layout(B, E / cluster, r).total; }

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const size_t smem = append_smem_bytes(a.B, a.E, a.r, a.cluster);
  cudaError_t e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.cluster, 2 * a.H, 1);
  cfg.blockDim = dim3(kAppendThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, append_kernel, a);
}

}  // namespace wsvd
