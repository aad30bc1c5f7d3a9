// Latent append for sm_100a: rotate the new token's activation with the block
// Hadamard S1, project it through A_Kh / A_Vh and quantise each (b, h, K|V)
// row into the cache (WSVD summaries: German §2.A for the per-head projection
// W_Kh ~= A_Kh . B_Kh, German §2.C for the Hadamard rotation S1 and the
// W8A8 / W8A4 quantisation).
//
// The work is a GEMV [B x E] . [E x r] per (h, K|V) unit, bound by reading A
// (2 * H * E * r fp16).  Each unit is split over a thread-block cluster of
// up to 8 CTAs along E.  Every CTA pulls its slice of x and then its
// contiguous A slice with 1-D bulk copies (TMA, no multicast), rotates its x
// slice with a fast Walsh-Hadamard transform (one warp per block, warp-level
// sync only) while A is in flight, and reduces its slice to a partial
// c[B][r].  Non-leader CTAs store their partial straight into the leader's
// shared memory (distributed shared memory) and arrive on the leader's
// mbarrier; the leader sums the slots in rank order (deterministic),
// quantises and writes the row.  The last leader to finish (a completion
// counter in the caller's workspace, reset to zero by that leader) advances
// seq_lens.
#include <cooperative_groups.h>

#include <map>
#include <mutex>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace wsvd {

constexpr int kAppendThreads = 256;
constexpr int kAppendWarps = kAppendThreads / 32;

struct AppendSmem {
  size_t a_off, xr_off, xs_off, slot_off, red_off, codes_off, bar_off, total;
};

static __host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A slice | raw x slice | rotated x (fp32) | partial slots [cluster][B][r] | reduction scratch | codes | barriers
static __host__ __device__ inline AppendSmem append_layout(int B, int Ec, int r, int cluster) {
  AppendSmem s;
  size_t o = 0;
  s.a_off = o;
  o = align_up(o + (size_t)Ec * r * 2, 128);
  s.xr_off = o;
  o = align_up(o + (size_t)B * Ec * 2, 128);
  s.xs_off = o;
  o = align_up(o + (size_t)B * Ec * 4, 16);
  s.slot_off = o;
  o = align_up(o + (size_t)cluster * B * r * 4, 16);
  s.red_off = o;
  o = align_up(o + (size_t)kAppendWarps * 4 * r * 4, 16);
  s.codes_off = o;
  o = align_up(o + (size_t)B * r, 16);
  s.bar_off = o;
  o += 3 * 8;
  s.total = align_up(o, 16);
  return s;
}

// The cluster's partials: slot[rank][b][j] in the leader's shared memory.
template <int BB>
__device__ __forceinline__ void gemv_slice(const __half* As, const float* xs, int B, int Ec, int r, float* red,
                                           float* dst /* [B][r], any shared window */, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  const int ncg = r / 8, nrg = kAppendThreads / ncg;
  const int cgi = tid % ncg, rg = tid / ncg;
  for (int bb0 = 0; bb0 < B; bb0 += BB) {
    float acc[BB][8];
#pragma unroll
    for (int bi = 0; bi < BB; ++bi)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[bi][k] = 0.f;
    for (int e = rg; e < Ec; e += nrg) {
      const uint4 av = *reinterpret_cast<const uint4*>(As + (size_t)e * r + cgi * 8);
      const float2 a01 = h2_pair(av.x), a23 = h2_pair(av.y), a45 = h2_pair(av.z), a67 = h2_pair(av.w);
      const float af[8] = {a01.x, a01.y, a23.x, a23.y, a45.x, a45.y, a67.x, a67.y};
#pragma unroll
      for (int bi = 0; bi < BB; ++bi) {
        const float xv = (bb0 + bi < B) ? xs[(size_t)(bb0 + bi) * Ec + e] : 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[bi][k] = fmaf(xv, af[k], acc[bi][k]);
      }
    }
    for (int o = ncg; o < 32; o <<= 1)
#pragma unroll
      for (int bi = 0; bi < BB; ++bi)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[bi][k] += __shfl_xor_sync(0xffffffffu, acc[bi][k], o);
    if (lane < ncg) {
#pragma unroll
      for (int bi = 0; bi < BB; ++bi)
#pragma unroll
        for (int k = 0; k < 8; ++k) red[(warp * BB + bi) * r + lane * 8 + k] = acc[bi][k];
    }
    __syncthreads();
    for (int idx = tid; idx < BB * r; idx += kAppendThreads) {
      const int bi = idx / r, j = idx % r;
      if (bb0 + bi < B) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kAppendWarps; ++w) s += red[(w * BB + bi) * r + j];
        dst[(size_t)(bb0 + bi) * r + j] = s;
      }
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.y, h = unit >> 1, kv = unit & 1;
  const int B = a.B, r = a.r, E = a.E;
  const int Ec = E / a.cluster, e0 = rank * Ec;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const AppendSmem L = append_layout(B, Ec, r, a.cluster);

  extern __shared__ __align__(128) uint8_t smem[];
  const __half* As = reinterpret_cast<const __half*>(smem + L.a_off);
  const uint16_t* xr = reinterpret_cast<const uint16_t*>(smem + L.xr_off);
  float* xs = reinterpret_cast<float*>(smem + L.xs_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  int8_t* codes = reinterpret_cast<int8_t*>(smem + L.codes_off);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* bar_a = bar_x + 1;
  uint64_t* bar_red = bar_x + 2;  // leader only: one arrival per non-leader CTA

  // 1. x slice first, then the A slice, on their way.
  if (tid == 0) {
    mbar_init(bar_x, 1);
    mbar_init(bar_a, 1);
    mbar_init(bar_red, a.cluster > 1 ? a.cluster - 1 : 1);
    fence_mbar_init();
    const uint64_t keep = l2_evict_last_policy(), once = l2_evict_first_policy();
    const uint32_t xrow = (uint32_t)Ec * 2;
    mbar_arrive_expect_tx(bar_x, xrow * B);
    for (int b = 0; b < B; ++b)
      bulk_g2s(smem + L.xr_off + (size_t)b * xrow, static_cast<const uint16_t*>(a.x) + (size_t)b * E + e0, xrow,
               bar_x, keep);
    const uint8_t* src = reinterpret_cast<const uint8_t*>((kv ? a.Av : a.Ak) + ((size_t)h * E + e0) * (size_t)r);
    const uint32_t bytes = (uint32_t)Ec * r * 2;
    mbar_arrive_expect_tx(bar_a, bytes);
    constexpr uint32_t kPiece = 32768;
    for (uint32_t off = 0; off < bytes; off += kPiece)
      bulk_g2s(smem + L.a_off + off, src + off, min(kPiece, bytes - off), bar_a, once);
  }
  // Every CTA's barriers are initialised before any remote access; the wait is
  // deferred until the first access so the barrier latency overlaps the copies.
  cluster.barrier_arrive();

  // 2. Rotate x: one warp per Hadamard block, butterflies with warp-level sync.
  if (!mbar_wait_bounded(bar_x, 0) && tid == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
  const int nblk = B * (Ec / a.blk);
  for (int blk = warp; blk < nblk; blk += kAppendWarps) {
    const int b = blk / (Ec / a.blk), off = (blk % (Ec / a.blk)) * a.blk;
    const uint16_t* src = xr + (size_t)b * Ec + off;
    float* dst = xs + (size_t)b * Ec + off;
    for (int i = lane; i < a.blk; i += 32)
      dst[i] = (a.x_dtype == WSVD_DTYPE_BF16) ? __uint_as_float((uint32_t)src[i] << 16)
                                              : __half2float(__ushort_as_half(src[i]));
    __syncwarp();
    for (int hh = 1; hh < a.blk; hh <<= 1) {
      for (int q = lane; q < a.blk / 2; q += 32) {
        const int i = (q / hh) * 2 * hh + (q % hh);
        const float u = dst[i], v = dst[i + hh];
        dst[i] = u + v;
        dst[i + hh] = u - v;
      }
      __syncwarp();
    }
  }
  __syncthreads();

  // 3. Wait for A (bounded), then the slice GEMV into this rank's slot of the leader.
  if (!mbar_wait_bounded(bar_a, 0) && tid == 0) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
  cluster.barrier_wait();
  float* my_slot = cluster.map_shared_rank(slots, 0) + (size_t)rank * B * r;
  if (B == 1) gemv_slice<1>(As, xs, B, Ec, r, red, my_slot, tid);
  else if (B == 2) gemv_slice<2>(As, xs, B, Ec, r, red, my_slot, tid);
  else gemv_slice<4>(As, xs, B, Ec, r, red, my_slot, tid);

  if (rank != 0) {
    // Publish the slot (release at cluster scope) and arrive on the leader's barrier.
    if (tid == 0) {
      asm volatile("fence.acq_rel.cluster;" ::: "memory");
      const uint32_t remote = static_cast<uint32_t>(__cvta_generic_to_shared(bar_red));
      uint32_t rbar;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(remote), "r"(0));
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rbar) : "memory");
    }
    return;
  }

  // 4. Leader: wait for the other ranks, sum the slots in rank order, quantise.
  if (a.cluster > 1) {
    bool ok = true;
    if (tid == 0) {
      const uint32_t addr = smem_u32(bar_red);
      const uint64_t t0 = globaltimer_ns();
      for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr)
            : "memory");
        if (done) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
      if (!ok) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
    }
    __syncthreads();
  }
  float* cfin = red;  // [B][r]
  for (int idx = tid; idx < B * r; idx += kAppendThreads) {
    float s = 0.f;
    for (int q = 0; q < a.cluster; ++q) s += slots[(size_t)q * B * r + idx];
    cfin[idx] = s * a.hnorm;
  }
  __syncthreads();
  const int Q = (a.bits == 8) ? 127 : 7;
  const int RB = r * a.bits / 8;
  for (int b = warp; b < B; b += kAppendWarps) {
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
      uint32_t* dstw = reinterpret_cast<uint32_t*>((kv ? a.lat_v : a.lat_k) + row * RB);
      for (int wi = lane; wi < RB / 4; wi += 32) {
        uint32_t word = 0;
        if (a.bits == 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) word |= (uint32_t)(uint8_t)codes[b * r + 4 * wi + k] << (8 * k);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) word |= ((uint32_t)codes[b * r + 8 * wi + k] & 0xFu) << (4 * k);
        }
        dstw[wi] = word;
      }
      if (lane == 0) (kv ? a.scale_v : a.scale_k)[row] = sh;
    } else if (lane == 0 && unit == 0) {
      set_err(a.err, WSVD_DEVERR_CACHE_FULL);
    }
  }
  __syncthreads();

  // 5. The last leader to finish advances the lengths.
  if (tid == 0) {
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
    if (E % (cl * blk) == 0 && (E / cl) % 8 == 0) return cl;
  return 0;
}

size_t append_smem_bytes(int B, int E, int r, int cluster) {
  return append_layout(B, E / cluster, r, cluster).total;
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const size_t smem = append_smem_bytes(a.B, a.E, a.r, a.cluster);
  {
    // Opt in to the dynamic shared memory once per device and size.
    static std::mutex mu;
    static std::map<int, size_t> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(dev);
    if (it == done.end() || it->second < smem) {
      e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      done[dev] = smem;
    }
  }
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
