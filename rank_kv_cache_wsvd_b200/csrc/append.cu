// Latent append for sm_100a: rotate the new token's activation with the block
// Hadamard S1, project it through A_Kh / A_Vh and quantise each (b, h, K|V)
// row into the cache (WSVD summaries: German §2.A for the per-head projection
// W_Kh ~= A_Kh . B_Kh, German §2.C for the Hadamard rotation S1 and the
// W8A8 / W8A4 quantisation).
//
// The work is a GEMV [B x E] . [E x r] per (h, K|V) unit, bound by reading A
// (2 * H * E * r fp16) once.  Each unit is split over a thread-block cluster
// of up to 8 CTAs along E.  Order of work in a CTA, chosen so that the A
// stream starts at once and nothing waits behind it:
//   1. plain loads of the CTA's x slice (small, L2-resident after the first
//      CTA), then the first 8 A rows of every thread are put in flight with
//      16-byte cp.async copies into a per-thread ring in shared memory;
//   2. the x slice is rotated (fast Walsh-Hadamard transform: in registers
//      and warp shuffles for blocks up to 128, shared-memory butterflies
//      beyond) while A arrives;
//   3. each thread consumes its ring slot by slot (cp.async.wait_group keeps 7
//      rows in flight) accumulating c[b][8 columns] in registers;
//   4. partials are reduced across the CTA (shuffles, then shared memory) and
//      stored into the cluster leader's shared memory with st.async stores
//      whose bytes complete on the leader's mbarrier; the leader sums the
//      ranks in order (deterministic), quantises with one warp per batch row
//      and writes the row.  The last leader to finish (a completion counter
//      in the caller's workspace, reset to zero by that leader) advances
//      seq_lens.
// A thread only ever reads ring slots it filled itself, so the ring needs no
// block-wide synchronisation.
#include <cooperative_groups.h>

#include <map>
#include <mutex>

#include "append_core.cuh"
#include "common.cuh"

namespace cg = cooperative_groups;

namespace wsvd {

struct AppendSmem {
  size_t ring_off, xs_off, slot_off, red_off, pos_off, bar_off, total;
};

static __host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ring [kRing][threads] x 16 B | rotated x (fp32) [B][Ec] | partial slots [cluster][B][r]
// | reduction scratch [warps][4][r] | row positions [16] | barrier
static __host__ __device__ inline AppendSmem append_layout(int B, int Ec, int r, int cluster) {
  AppendSmem s;
  size_t o = 0;
  s.ring_off = o;
  o += (size_t)kRing * kAppendThreads * 16;
  s.xs_off = o;
  o = align_up(o + (size_t)B * Ec * 4, 16);
  s.slot_off = o;
  o = align_up(o + (size_t)cluster * B * r * 4, 16);
  s.red_off = o;
  o = align_up(o + (size_t)kAppendWarps * 4 * r * 4, 16);
  s.pos_off = o;
  o += 16 * 4;
  s.bar_off = o;
  o += 8;
  s.total = align_up(o, 16);
  return s;
}

// R: the latent width, a compile-time constant of each instantiation.
template <int BB, bool W8, int R>
__device__ __forceinline__ void append_body(const AppendArgs& a, cg::cluster_group& cluster, uint8_t* smem,
                                            const AppendSmem& L) {
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.y, h = unit >> 1, kv = unit & 1;
  constexpr int r = R;
  const int B = a.B, E = a.E;
  const int Ec = E / a.cluster, e0 = rank * Ec;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint4* ring = reinterpret_cast<uint4*>(smem + L.ring_off);
  float* xs = reinterpret_cast<float*>(smem + L.xs_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  // Leader: completes when every other rank's slot values have landed
  // (transaction bytes of their st.async stores).
  uint64_t* bar_red = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  int* pos_sm = reinterpret_cast<int*>(smem + L.pos_off);  // leader: seq_lens[b] as read at launch

  // int8 weights: the leader's quantising lanes load their column scales now.
  ColScales<R> cs;
  if (W8 && rank == 0) cs.load((kv ? a.sAv : a.sAk) + (size_t)h * r, r, lane);
  // The leader reads the row positions first so that their latency is hidden.
  // No CTA writes seq_lens before every leader has counted itself done (below).
  if (rank == 0 && tid < B) pos_sm[tid] = ld_relaxed_gpu(a.seq_lens + tid);
  if (tid == 0) {
    mbar_init(bar_red, 1);
    fence_mbar_init();
    if (rank == 0 && a.cluster > 1) mbar_arrive_expect_tx(bar_red, (uint32_t)((a.cluster - 1) * B * r * 4));
  }
  // Every CTA's barrier is initialised before any remote access; the wait is
  // deferred to the first remote access.
  cluster_arrive_relaxed();

  // 1. x slice loads first (registers), then the A stream.  Behind the grid
  // that writes x, the A stream goes first and x is read after the wait.
  const bool fast = x_fast_path(B, Ec, a.blk);
  uint2 xraw[kXChunks];
  if (!a.dep && fast) load_x_slice(xraw, a.x, B, E, e0, Ec, warp, lane);
  const int ncg = r / 8, nrg = kAppendThreads / ncg;
  RowWalk<W8> w;
  w.A = static_cast<const uint8_t*>(kv ? a.Av : a.Ak) + ((size_t)h * E + e0) * (size_t)r * (W8 ? 1 : 2);
  w.r = r; w.Ec = Ec; w.nrg = nrg; w.rg = tid / ncg; w.cgi = tid % ncg;
  w.nrows = w.rg < Ec ? (Ec - 1 - w.rg) / nrg + 1 : 0;
#pragma unroll 1
  for (int k = 0; k < kRing; ++k) w.issue(ring, k, tid);
  if (a.dep) {
    griddep_wait();
    if (fast) load_x_slice(xraw, a.x, B, E, e0, Ec, warp, lane);
  }

  // 2. Rotate x into xs[b][e] (unnormalised; 1/sqrt(blk) is applied to c).
  auto block_sync = []() { __syncthreads(); };
  rotate_x_slice(fast, xraw, xs, a.x, a.x_dtype, B, E, e0, Ec, a.blk, tid, block_sync);

  // 3. + 4. Stream the A rows, reduce into this rank's slot of the leader.
  cluster_wait();
  const uint32_t remote_slot = rank ? mapa_shared(slots + (size_t)rank * B * r, 0) : 0u;
  const uint32_t remote_bar = rank ? mapa_shared(bar_red, 0) : 0u;
  for (int bb0 = 0; bb0 < B; bb0 += BB) {
    if (bb0 > 0) {
#pragma unroll 1
      for (int k = 0; k < kRing; ++k) w.issue(ring, k, tid);  // re-stream (L2) for the next batch rows
    }
    float2 acc[BB][4];
    stream_rows<BB, W8>(w, ring, xs, B, bb0, acc, tid);
    reduce_cta<BB, R / 8>(acc, r, min(BB, B - bb0), red, slots + (size_t)bb0 * r, remote_slot + 4u * bb0 * r,
                          remote_bar, tid, block_sync);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  // The A stream is done: a decode launched behind this kernel may now be
  // scheduled (it reads q and its B matrices, and waits for this grid to
  // complete before it touches the cache).  Triggering here rather than at
  // launch lets the non-leader CTAs leave first, so the decode's clusters
  // find whole SMs.
  griddep_launch_dependents();
  if (rank != 0) return;  // slot values are in flight to the leader

  // 5. Leader: wait for the other ranks, sum the slots in rank order, quantise
  //    (one warp per batch row; lane owns columns j = lane + 32k).
  if (a.cluster > 1) {
    if (tid == 0 && !mbar_wait_cluster_bounded(bar_red, 0)) set_err(a.err, WSVD_DEVERR_PIPE_TIMEOUT);
  }
  __syncthreads();  // slots landed; pos_sm visible
  // 6. Completion counter, overlapping the quantisation below: this CTA's only
  //    reads of seq_lens (at launch) are ordered before its add (acq_rel after
  //    the CTA barrier), so the last leader may advance the lengths at once.
  //    The row stores need no ordering with it: later kernels see both.
  if (tid == kAppendThreads - 32) {
    const int prev = atom_add_acq_rel_gpu(a.counter, 1);
    if (prev == (int)gridDim.y - 1) {
      for (int b = 0; b < B; ++b) {
        const int pos = pos_sm[b];
        if (pos >= 0 && pos < a.L_cap) st_relaxed_gpu(a.seq_lens + b, pos + 1);
      }
      st_relaxed_gpu(a.counter, 0);
    }
  }
  const int RB = r * a.bits / 8;
  for (int b = warp; b < B; b += kAppendWarps) {
    const int pos = pos_sm[b];
    const bool ok = pos >= 0 && pos < a.L_cap;
    const size_t row = ((size_t)b * a.H + h) * a.L_cap + (ok ? pos : 0);
    const __half sh = quantise_append_row<W8, R>(slots + (size_t)b * r, (size_t)B * r, a.cluster, r, a.bits, a.hnorm,
                                                 cs, ok, (kv ? a.lat_v : a.lat_k) + row * RB, nullptr, lane);
    if (lane == 0) {
      if (ok) (kv ? a.scale_v : a.scale_k)[row] = sh;
      else if (unit == 0) set_err(a.err, WSVD_DEVERR_CACHE_FULL);
    }
  }
}

// One kernel per weight format and latent width (r is 8, 16, 32, 64 or 128):
// each gets its own register allocation, the row walk, the reduction and the
// quantiser are fixed at compile time, and each kernel holds only its own
// bodies (a kernel with every width's bodies measured instruction-fetch
// stalls at thirteen cycles per issued instruction).
template <bool W8, int R>
__global__ void __launch_bounds__(kAppendThreads, 4) append_kernel(const AppendArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const AppendSmem L = append_layout(a.B, a.E / a.cluster, R, a.cluster);
  if (a.B == 1) append_body<1, W8, R>(a, cluster, smem, L);
  else if (a.B == 2) append_body<2, W8, R>(a, cluster, smem, L);
  else append_body<4, W8, R>(a, cluster, smem, L);
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
  void (*kern)(const AppendArgs) = nullptr;
  switch (a.r) {
    case 8: kern = a.w8 ? append_kernel<true, 8> : append_kernel<false, 8>; break;
    case 16: kern = a.w8 ? append_kernel<true, 16> : append_kernel<false, 16>; break;
    case 32: kern = a.w8 ? append_kernel<true, 32> : append_kernel<false, 32>; break;
    case 64: kern = a.w8 ? append_kernel<true, 64> : append_kernel<false, 64>; break;
    case 128: kern = a.w8 ? append_kernel<true, 128> : append_kernel<false, 128>; break;
    default: return cudaErrorInvalidValue;  // rejected by the argument checks before this
  }
  {
    // Opt in to the dynamic shared memory once per device, kernel and size.
    static std::mutex mu;
    static std::map<std::pair<int, const void*>, size_t> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, reinterpret_cast<const void*>(kern));
    auto it = done.find(key);
    if (it == done.end() || it->second < smem) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      done[key] = smem;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.cluster, 2 * a.H, 1);
  cfg.blockDim = dim3(kAppendThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.dep ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace wsvd
