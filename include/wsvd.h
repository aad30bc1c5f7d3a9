/*
 * wsvd.h -- C ABI of the B200 (sm_100a) WSVD low-rank KV-cache decode library.
 *
 * The operations follow the WSVD summaries ("WSVD: Weighted Low-Rank
 * Approximation for Fast and Efficient Execution of Low-Precision
 * Vision-Language Models", gist.science paper 2604.02570):
 *   - per-head factorisation W_Kh ~= A_Kh . B_Kh, A_Kh in R^{E x r},
 *     B_Kh in R^{r x Hd}, and a per-head latent cache C_Kh of L x r values
 *     (Arabic summary §2.a; German summary §2.A "Fein granulare SVD pro
 *     Attention-Head");
 *   - low-precision latents (W8A8 / W8A4) with the Hadamard rotation S1 on the
 *     activations (German summary §2.C "Quantisierungsbewusstes Training");
 *   - a fused decode that rebuilds K/V from latent tiles on chip and runs
 *     q.K^T, softmax and the V product without writing K/V to memory
 *     (Japanese summary §2.4 "システム実装：融合カーネル"; German §2.D).
 *
 * Conventions for every entry point:
 *   - Array pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates, frees or synchronises; it launches on `stream` (a
 *     cudaStream_t passed as void*, NULL = legacy default stream) and returns.
 *   - 16-bit floats are passed as `const void*` (IEEE fp16 or bf16 bits).
 *   - All arrays are dense row-major in the shapes given; every array pointer
 *     must be 16-byte aligned.
 *   - Return value: a wsvd_status.  Argument problems found on the host are
 *     reported before anything is launched.  A launch failure returns
 *     WSVD_ERR_CUDA (cudaGetLastError).  Problems found on the device (a
 *     sequence length out of range, a full cache) never fault: the kernel ORs a
 *     WSVD_DEVERR_* bit into the caller's int32 `*err` (device memory; may be
 *     NULL) and treats the sequence as described per call.
 *   - Outputs are written in full on every successful launch.  Results are
 *     deterministic: the same inputs, shapes and device give the same bits.
 */
#ifndef WSVD_B200_H
#define WSVD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WSVD_OK = 0,
  WSVD_ERR_INVALID_ARG = 1,          /* null pointer, bad size, misaligned pointer */
  WSVD_ERR_UNSUPPORTED = 2,          /* valid but not built (e.g. row bytes not a multiple of 16) */
  WSVD_ERR_CUDA = 3,                 /* the CUDA runtime reported an error */
  WSVD_ERR_WORKSPACE_TOO_SMALL = 4   /* workspace_bytes below the matching *_workspace_size() */
} wsvd_status;

/* 16-bit float formats for q and x. */
enum { WSVD_DTYPE_FP16 = 0, WSVD_DTYPE_BF16 = 1 };

/* Bits ORed into the caller's device error word. */
enum {
  WSVD_DEVERR_LEN_RANGE = 1,     /* decode: seq_lens[b] < 0 or > L_cap; that sequence's output is 0 */
  WSVD_DEVERR_CACHE_FULL = 2,    /* append: seq_lens[b] >= L_cap (or < 0); row not written, length kept */
  WSVD_DEVERR_PIPE_TIMEOUT = 4   /* a pipeline wait exceeded its time limit; outputs are not valid */
};

/* Human-readable name of a wsvd_status. Never NULL. */
const char* wsvd_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
int wsvd_abi_version(void);

/* ---------------------------------------------------------------- footprint
 * Bytes of a per-head latent cache: K and V codes (L_cap x r per head, `bits`
 * per code) plus one fp16 scale per token per head for each
 * (Arabic summary §2.a: the latent footprint per head is L x r).            */
size_t wsvd_cache_bytes(int B, int H, int L_cap, int r, int bits);
/* Bytes of a conventional shared fp16 latent: L_cap x R for K and for V
 * (Arabic summary §2.a: the shared latent is L x R).                        */
size_t shared_cache_bytes(int B, int L_cap, int R);
/* Bytes of a dense fp16 K/V cache (L_cap x Hd per head, K and V).           */
size_t dense_cache_bytes(int B, int H, int L_cap, int Hd);

/* ---------------------------------------------------------------- WSVD decode
 * One decode step of attention over a per-head low-rank, low-precision cache
 * (Japanese §2.4 / German §2.D, the fused low-rank flash-decoding kernel).
 *
 * For each sequence b < B and head h < H, with n = seq_lens[b] tokens:
 *   lat_K[l] = code_K[b,h,l,:] * scale_k[b,h,l]      (l < n; likewise V)
 *   K = lat_K . B_k[h],  V = lat_V . B_v[h]          (n x Hd, never stored)
 *   out[b,h,:] = softmax(K . q[b,h,:] * softmax_scale) . V
 * computed in the reassociated form q' = B_k[h] . q, score_l = s_K,l
 * (code_K,l . q'), out = ((sum_l p_l s_V,l code_V,l) / sum_l p_l) . B_v[h],
 * fp32 accumulation.  A sequence with n = 0 gets out = 0.
 *
 *   B, H, Hd, r, bits : batch (<= 4096), heads, head dim (32, 64, 128 or 256), rank,
 *                       bits per code (8 or 4).  Row bytes r*bits/8 must be
 *                       16, 32, 64 or 128 for int8 and 16, 32 or 64 for int4
 *                       (else WSVD_ERR_UNSUPPORTED).
 *   L_cap             : rows per (b, h) in the cache; multiple of 8.
 *   seq_lens  [B]            int32: tokens used per sequence (0 <= n <= L_cap).
 *   q         [B][H][Hd]     fp16 or bf16 (q_dtype).
 *   lat_k, lat_v [B][H][L_cap][r*bits/8] uint8: int8 two's complement codes,
 *                            or int4 with element 2j in bits 0-3 and 2j+1 in
 *                            bits 4-7 of byte j (two's complement nibbles).
 *   scale_k, scale_v [B][H][L_cap] fp16 per-token scales.
 *   B_k, B_v  [H][r][Hd]     fp16.
 *   softmax_scale            0 selects 1/sqrt(Hd).
 *   out       [B][H][Hd]     float32, written.
 *   workspace                device scratch of at least
 *                            wsvd_decode_workspace_size(B, H, r) bytes that is
 *                            ZERO before the first call (cudaMemset once):
 *                            it holds split partials, one completion counter
 *                            per (b, h) and the projected queries q' [B][H][r]
 *                            fp32, and every call leaves the counters zero.
 *                            Calls that share a workspace must not overlap on
 *                            the GPU.
 *   err                      optional device int32; WSVD_DEVERR_LEN_RANGE.
 * Rows >= seq_lens[b] are never used: their bytes may hold anything.
 * Depending on the sizes, one call launches one kernel (one cluster of CTAs
 * per (b, h)) or two (q' for every (b, h), then the split-L grid launched
 * behind it as a programmatic dependent); wsvd_decode_launch_count tells
 * which, for the given sizes on the current device.                        */
size_t wsvd_decode_workspace_size(int B, int H, int r);
int wsvd_decode_launch_count(int B, int H, int Hd, int r, int bits, int L_cap);
int wsvd_decode_attention(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                          const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                          const void* scale_k, const void* scale_v, const void* B_k, const void* B_v,
                          float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                          int32_t* err, void* stream);

/* ---------------------------------------------------------------- grouped and multi-token decode
 * The decode of wsvd_decode_attention for several queries per latent head
 * (the fused low-rank decode of Japanese §2.4 / German §2.D, which the pages
 * describe for one query per head and token):
 *   - Hq query heads share Hkv latent heads (grouped-query attention):
 *     query head g reads latent head g / G, G = Hq / Hkv (consecutive query
 *     heads form a group), with that head's cache and factors;
 *   - Tq new tokens per sequence are decoded at once (a chunked or
 *     speculative step): they are the last Tq cached rows, and query token t
 *     of sequence b attends to rows [0, seq_lens[b] - Tq + 1 + t) (causal
 *     inside the block).  A query that sees no row gets out = 0.
 * Per query: out = softmax(K . q * softmax_scale) . V over its visible rows,
 * K = lat_K . B_k[h], V = lat_V . B_v[h] (h its latent head), computed
 * reassociated as in wsvd_decode_attention.  One tile of cached latents is
 * read once for all G * Tq queries of its latent head; the score and value
 * products run on the tensor cores (int8 scores against a 24-bit fixed-point
 * q'; values in fp16 hi + lo halves with fp32 accumulation).
 *
 *   q         [B][Tq][Hq][Hd] fp16 or bf16 (wsvd_decode_gqa: [B][Hq][Hd]).
 *   lat_k, lat_v [B][Hkv][L_cap][r*bits/8], scale_k, scale_v [B][Hkv][L_cap],
 *             B_k, B_v [Hkv][r][Hd]: formats as for wsvd_decode_attention.
 *   out       [B][Tq][Hq][Hd] float32 (wsvd_decode_gqa: [B][Hq][Hd]).
 *   Hq a multiple of Hkv; G * Tq <= 64; Hd in {32, 64, 128, 256}; row bytes
 *   r*bits/8 in {16, 32, 64} (int8 r = 16, 32, 64; int4 r = 32, 64, 128);
 *   L_cap a multiple of 8; B <= 65535.  Else WSVD_ERR_UNSUPPORTED.
 *   workspace  at least wsvd_decode_multi_workspace_size(...) bytes, ZERO
 *             before the first call; it holds split partials and one counter
 *             per (sequence, latent head, group of 16 queries); every call
 *             leaves the counters zero.  Calls sharing it must not overlap.
 *   err        optional; WSVD_DEVERR_LEN_RANGE as for wsvd_decode_attention.
 * One launch per call.                                                       */
size_t wsvd_decode_multi_workspace_size(int B, int Tq, int Hq, int Hkv, int r, int L_cap);
int wsvd_decode_multi(int B, int Tq, int Hq, int Hkv, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                      const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                      const void* scale_v, const void* B_k, const void* B_v, float softmax_scale, float* out,
                      void* workspace, size_t workspace_bytes, int32_t* err, void* stream);
/* wsvd_decode_multi with Tq = 1.                                            */
size_t wsvd_decode_gqa_workspace_size(int B, int Hq, int Hkv, int r, int L_cap);
int wsvd_decode_gqa(int B, int Hq, int Hkv, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                    const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                    const void* scale_v, const void* B_k, const void* B_v, float softmax_scale, float* out,
                    void* workspace, size_t workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- WSVD decode without allocation
 * The WSVD summaries have no counterpart to this entry point: it is a
 * deployment convenience of this library.
 *
 * Same operation, arguments and results as wsvd_decode_attention, for callers
 * that cannot call cudaMalloc: a serving runtime whose device memory is one
 * pre-sized pool owned by another allocator, code that runs where a device
 * allocation would synchronise the device or fail (inside latency-critical
 * loops, under memory limits), or a host language binding without access to
 * device allocation.  The scratch it needs (split partials and one counter
 * per (b, h), the projected queries) lives in a static device array of WSVD_NOALLOC_SCRATCH_BYTES
 * that every GPU loading the library holds until the process exits; the call
 * itself allocates nothing.
 *   - A problem whose scratch need, wsvd_decode_workspace_size(B, H, r),
 *     exceeds WSVD_NOALLOC_SCRATCH_BYTES is rejected with
 *     WSVD_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture.
 *   - Arguments are validated as by wsvd_decode_attention, in the same
 *     order, before anything is queued on `stream`; then the call clears the
 *     per-(b, h) counters (an asynchronous memset of 4 * B * H bytes on
 *     `stream`) and launches the decode.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other threads) race and give wrong results.                  */
#define WSVD_NOALLOC_SCRATCH_BYTES (2u << 20)
int wsvd_decode_attention_noalloc(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                                  const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                                  const void* scale_k, const void* scale_v, const void* B_k, const void* B_v,
                                  float softmax_scale, float* out, int32_t* err, void* stream);

/* ---------------------------------------------------------------- latent append
 * Writes one new token per sequence into the latent cache (the projection of
 * the new token through A_Kh / A_Vh, German §2.A, after the Hadamard rotation
 * S1 of German §2.C), then advances its length:
 *   x~ = x[b,:] . blockdiag(H_blk / sqrt(blk))   (Sylvester order, blk = hadamard_block)
 *   c_K = x~ . A_k[h],  c_V = x~ . A_v[h]         (r values each, fp32)
 *   per (b, h, K|V): scale = fp16(max_j |c_j| / Q)  (Q = 127 int8, 7 int4),
 *   code_j = clamp(round_half_even(c_j / scale), -Q, Q) (scale 0 -> codes 0);
 *   row seq_lens[b] of lat_k/lat_v/scale_k/scale_v is written, then
 *   seq_lens[b] += 1.
 * A sequence with seq_lens[b] >= L_cap (or < 0) is not written and not
 * advanced; WSVD_DEVERR_CACHE_FULL is raised.
 *
 *   x          [B][E]       bf16 or fp16 (x_dtype); E % hadamard_block == 0.
 *   A_k, A_v   [H][E][r]    fp16.
 *   hadamard_block          power of two in [2, 1024] (1 = no rotation).
 *   E                       multiple of hadamard_block and of 8, at most
 *                           65536.  E is split along a cluster of up to 8
 *                           CTAs (the largest c in {8,4,2,1} with
 *                           E % (c * hadamard_block) == 0 and (E/c) % 8 == 0);
 *                           WSVD_ERR_UNSUPPORTED when the rotated slice,
 *                           B * E/c fp32 values, and the 32 KB row ring do
 *                           not fit in 200 KB of shared memory.
 *   r                       8, 16, 32, 64 or 128.
 *   B                       1..16.
 *   seq_lens   [B]          int32, read and advanced in place.
 *   workspace               at least wsvd_append_workspace_size() bytes of
 *                           device memory that is ZERO before the first call
 *                           (cudaMemset once); every call leaves it zero.
 *                           Calls that share a workspace must not overlap.
 * Rows other than seq_lens[b] are never written.                             */
size_t wsvd_append_workspace_size(void);
int wsvd_latent_append(int B, int H, int E, int r, int bits, int L_cap, int hadamard_block,
                       const void* x, int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens,
                       uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, void* workspace,
                       size_t workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- prefill latent write
 * Writes a block of T new tokens per sequence (a prompt, e.g. the image tokens
 * of a vision-language prompt) into the latent cache in one call: token t of
 * sequence b is rotated, projected and quantised as by wsvd_latent_append
 * (German §2.A projection, German §2.C rotation S1 and W8A8 / W8A4 quantiser)
 * and stored at row seq_lens[b] + t; then seq_lens[b] += T.  The pages give
 * no block interface; the rows written are those of T successive appends.
 * A sequence with seq_lens[b] < 0 or seq_lens[b] + T > L_cap is not written
 * and not advanced; WSVD_DEVERR_CACHE_FULL is raised.
 * The projection runs as a GEMM on the tensor cores: the rotated activations
 * are split into two fp16 halves (hi + lo, 22 significant bits after an exact
 * per-token power-of-two scaling), each multiplied by the fp16 weights with
 * fp32 accumulation.
 *
 *   x          [B][T][E]    bf16 or fp16 (x_dtype); the rotated values times
 *                           their power-of-two scale must stay finite in fp16
 *                           (any finite bf16 input does).
 *   A_k, A_v   [H][E][r]    fp16.
 *   hadamard_block          power of two in [1, 1024], E % hadamard_block == 0.
 *   E                       multiple of 64, at most 16384.
 *   r                       8, 16, 32, 64 or 128.
 *   seq_lens   [B]          int32, read and advanced in place.
 *   workspace               at least wsvd_prefill_workspace_size(B, T, E)
 *                           bytes (the split rotated activations; no zeroing
 *                           needed).  Calls that share it must not overlap.
 * T = 0 (or B = 0) launches nothing.  Three launches otherwise (rotate,
 * GEMM + quantiser, length advance), all on `stream`.                       */
size_t wsvd_prefill_workspace_size(int B, int T, int E);
int wsvd_latent_prefill(int B, int T, int H, int E, int r, int bits, int L_cap, int hadamard_block,
                        const void* x, int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens,
                        uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, void* workspace,
                        size_t workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- one decode step
 * wsvd_latent_append followed by wsvd_decode_attention on the same stream: the
 * decode step of the method (append the new token's latents, then attend over
 * the cache including it; WSVD summaries, German §2.A and §2.C).  The pages
 * define no separate interface for it; the results are those of the two calls
 * made back to back, bit for bit.
 * For one sequence (B = 1) whose decode takes the one-cluster-per-head path
 * with the append's cluster size (short caches: each of the cluster's ranks
 * holds at most one tile of rows), one kernel does both: cluster h projects
 * head h's new K and V rows, the rank whose rows hold the new token quantises
 * them, writes them to the cache and attends over them, and the other ranks
 * attend over their rows meanwhile.  Otherwise the decode is launched as a
 * programmatic dependent of the append: its launch and its query projection
 * q' = B_Kh . q overlap the append, and it reads seq_lens and the cache only
 * after the append grid has completed.  Either way q, B_k and B_v must
 * already be final when this call is made (they are read while the append
 * runs; the append itself never writes them).  wsvd_step_launch_count tells
 * how many kernels a step takes for the given sizes on the current device.
 *   append_workspace   wsvd_append_workspace_size() bytes, contract as for
 *                      wsvd_latent_append;
 *   decode_workspace   wsvd_decode_workspace_size(B, H, r) bytes, contract as
 *                      for wsvd_decode_attention.
 * Every argument of both operations is validated before anything is launched;
 * the status codes are those of the two calls.                              */
int wsvd_step_launch_count(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block, int w8);
int wsvd_append_and_decode(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                           const void* x, int x_dtype, const void* A_k, const void* A_v, int32_t* seq_lens,
                           uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v, const void* q,
                           int q_dtype, const void* B_k, const void* B_v, float softmax_scale, float* out,
                           void* append_workspace, size_t append_workspace_bytes, void* decode_workspace,
                           size_t decode_workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- one decode step from host buffers
 * wsvd_append_and_decode for a caller whose per-step inputs and output live in
 * host memory (a serving loop that receives the new token's activation and
 * query from the host and returns the attention output there).  The pages
 * have no counterpart: it exists so that one library call covers a whole
 * step, host transfers included.  On `stream`, in order:
 *   x_host [B][E] and q_host [B][H][Hd] (16-bit, x_dtype / q_dtype) are
 *   brought into step_workspace; the append and the decode run as in
 *   wsvd_append_and_decode on those device copies; out [B][H][Hd] fp32 is
 *   delivered to out_host.
 * How the bytes move depends on the host memory:
 *   - x_host, q_host and out_host all page-locked and mapped into the device's
 *     address space (every cudaHostAlloc / cudaMallocHost allocation under
 *     unified addressing), 16-byte aligned, with B*E*2 and B*H*Hd*2 multiples
 *     of 16: a small kernel reads x and q from host memory (the append is
 *     launched behind it as a programmatic dependent and streams A_k, A_v in
 *     the meantime), and the decode stores out straight into out_host.  No
 *     copy-engine transfer is queued.
 *   - otherwise: cudaMemcpyAsync copies in and out (pageable memory goes
 *     through the driver's staging).
 * The call returns once everything is queued; out_host is valid after the
 * stream is synchronised, and the host may rewrite x_host and q_host only
 * after that (they are read while the step runs).
 *   step_workspace   device memory of at least
 *                    wsvd_step_host_workspace_size(B, H, Hd, E, r) bytes that is
 *                    ZERO before the first call; it holds the append and
 *                    decode workspaces (their counters are left zero) and the
 *                    device copies of x, q (and out, for the copy route).
 *                    Calls that share it must not overlap on the GPU.
 * Every other argument is as for wsvd_append_and_decode (device pointers).
 * All arguments are validated before anything is queued.                    */
size_t wsvd_step_host_workspace_size(int B, int H, int Hd, int E, int r);
int wsvd_append_and_decode_host(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                                const void* x_host, int x_dtype, const void* A_k, const void* A_v,
                                int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                                const void* q_host, int q_dtype, const void* B_k, const void* B_v,
                                float softmax_scale, float* out_host, void* step_workspace,
                                size_t step_workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- the host-buffer step as one graph
 * The launches of one wsvd_append_and_decode_host call captured once into a
 * CUDA graph, replayed per step with one cudaGraphLaunch (a serving loop's
 * per-step cost is then one call, and the device runs the step's three
 * kernels without waiting for the host between them).  The pages have no
 * counterpart.
 * wsvd_step_host_graph_create takes the arguments of
 * wsvd_append_and_decode_host (minus the stream) and binds them: every
 * pointer, the shapes and softmax_scale are fixed in the graph, so each launch
 * reads the host buffers' current contents and the device state (seq_lens,
 * the cache) as it is at that point in the stream.  It validates exactly as
 * wsvd_append_and_decode_host does and runs nothing on the GPU.  It needs
 * the in-place route (x_host, q_host, out_host pinned, mapped and aligned as
 * described there) and returns WSVD_ERR_UNSUPPORTED otherwise.  On success
 * *graph receives a handle; on failure it is set to NULL.
 * wsvd_step_host_graph_launch queues one step on `stream` (WSVD_ERR_INVALID_ARG
 * for a NULL handle, WSVD_ERR_CUDA if the launch fails).  Launches of one
 * handle must not overlap on the GPU (they share the step workspace).
 * wsvd_step_host_graph_destroy releases the handle (NULL is ignored); no
 * launch of it may still be pending.                                          */
typedef struct wsvd_step_graph wsvd_step_graph;
int wsvd_step_host_graph_create(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                                const void* x_host, int x_dtype, const void* A_k, const void* A_v,
                                int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                                const void* q_host, int q_dtype, const void* B_k, const void* B_v,
                                float softmax_scale, float* out_host, void* step_workspace,
                                size_t step_workspace_bytes, int32_t* err, wsvd_step_graph** graph);
int wsvd_step_host_graph_launch(wsvd_step_graph* graph, void* stream);
void wsvd_step_host_graph_destroy(wsvd_step_graph* graph);

/* ---------------------------------------------------------------- int8 weights (W8)
 * The same three operations with the low-rank factors stored as int8 weights
 * (the "W8" of the method's W8A8 / W8A4 configurations, German §2.C): every
 * weight matrix has one fp32 scale per output column,
 *   A_h[e][j] = A_k[h][e][j] * sA_k[h][j]   (A_k, A_v  [H][E][r] int8, sA_* [H][r]  fp32),
 *   B_h[j][d] = B_k[h][j][d] * sB_k[h][d]   (B_k, B_v  [H][r][Hd] int8, sB_* [H][Hd] fp32),
 * and the results are those of the fp16 entry points given those dequantised
 * weights (the kernels fold each scale in once: into q for B_k, after the
 * column sums for A and B_v).  The pages fix no granularity for the weight
 * scales; per output column is this library's reading.  Int8 matrices and
 * the B scales sB_k, sB_v must be 16-byte aligned (the decode stages a head's
 * rows of them with bulk copies; else WSVD_ERR_INVALID_ARG); the A scales are
 * read with plain loads.  Every other argument, the workspace contracts and
 * the status codes are those of the fp16 entry points. */
int wsvd_decode_attention_w8(int B, int H, int Hd, int r, int bits, int L_cap, const int32_t* seq_lens,
                             const void* q, int q_dtype, const uint8_t* lat_k, const uint8_t* lat_v,
                             const void* scale_k, const void* scale_v, const int8_t* B_k, const int8_t* B_v,
                             const float* sB_k, const float* sB_v, float softmax_scale, float* out, void* workspace,
                             size_t workspace_bytes, int32_t* err, void* stream);
int wsvd_latent_append_w8(int B, int H, int E, int r, int bits, int L_cap, int hadamard_block, const void* x,
                          int x_dtype, const int8_t* A_k, const int8_t* A_v, const float* sA_k, const float* sA_v,
                          int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k, void* scale_v,
                          void* workspace, size_t workspace_bytes, int32_t* err, void* stream);
int wsvd_append_and_decode_w8(int B, int H, int Hd, int E, int r, int bits, int L_cap, int hadamard_block,
                              const void* x, int x_dtype, const int8_t* A_k, const int8_t* A_v, const float* sA_k,
                              const float* sA_v, int32_t* seq_lens, uint8_t* lat_k, uint8_t* lat_v, void* scale_k,
                              void* scale_v, const void* q, int q_dtype, const int8_t* B_k, const int8_t* B_v,
                              const float* sB_k, const float* sB_v, float softmax_scale, float* out,
                              void* append_workspace, size_t append_workspace_bytes, void* decode_workspace,
                              size_t decode_workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- latent rotation S2 (weight preparation)
 * Folds an orthogonal rotation S2 of each head's latent space into the
 * low-rank factors (the "Outlier-Smoothing" transforms S1, S2 of the WSVD
 * summaries, German §2.C and Arabic §2.c; S2 is learned jointly with A and B,
 * and given here):
 *   A'_k[h] = A_k[h] . S2_k[h],   B'_k[h] = S2_k[h]^T . B_k[h]   (same for V).
 * With S2 . S2^T = I the rebuilt keys and values c . B are unchanged, while
 * the cache then holds the rotated latents c . S2, which are what the append
 * quantises.  Run once at model load; the other entry points take A', B'.
 *   S2_k, S2_v            [H][r][r] float32, orthogonal (not checked).
 *   A_k, A_v              [H][E][r] fp16;  A_k_out, A_v_out same shape, written.
 *   B_k, B_v              [H][r][Hd] fp16; B_k_out, B_v_out same shape, written.
 * fp32 dot products over r, each result rounded once to fp16.  No output may
 * share a byte with any input or with another output (WSVD_ERR_INVALID_ARG);
 * r <= 128, H <= 65535.  Launches four small kernels on `stream`.           */
int wsvd_fold_latent_rotation(int H, int E, int r, int Hd, const float* S2_k, const float* S2_v, const void* A_k,
                              const void* A_v, const void* B_k, const void* B_v, void* A_k_out, void* A_v_out,
                              void* B_k_out, void* B_v_out, void* stream);

/* ---------------------------------------------------------------- comparison: dense decode
 * The flash-decoding baseline the pages compare against (German §4
 * "Ergebnisse"): out[b,h] = softmax(K[b,h,:n] . q[b,h] * softmax_scale) . V[b,h,:n]
 * over a dense fp16 cache.  K, V [B][H][L_cap][Hd] fp16 (Hd in {32, 64, 128, 256}).
 * Other arguments (workspace contract included) as for wsvd_decode_attention. */
size_t dense_decode_workspace_size(int B, int H, int Hd);
int dense_decode_attention(int B, int H, int Hd, int L_cap, const int32_t* seq_lens, const void* q,
                           int q_dtype, const void* K, const void* V, float softmax_scale, float* out,
                           void* workspace, size_t workspace_bytes, int32_t* err, void* stream);

/* ---------------------------------------------------------------- comparison: shared-latent SVD decode
 * The conventional SVD decode the pages measure against (Japanese §1, German
 * §1): one latent per sequence shared by all heads, lat_k, lat_v
 * [B][L_cap][R] fp16, and per-head up-projections B_k, B_v [H][R][Hd] fp16.
 * Every head reads the whole shared latent:
 *   K_h = lat_k[b,:n] . B_k[h], V_h = lat_v[b,:n] . B_v[h],
 *   out[b,h] = softmax(K_h . q[b,h] * softmax_scale) . V_h.
 * R in {128, 256, 512, 1024}.  Other arguments (workspace contract included)
 * as for wsvd_decode_attention.                                             */
size_t shared_decode_workspace_size(int B, int H, int R);
int shared_latent_svd_decode(int B, int H, int Hd, int R, int L_cap, const int32_t* seq_lens,
                             const void* q, int q_dtype, const void* lat_k, const void* lat_v,
                             const void* B_k, const void* B_v, float softmax_scale, float* out,
                             void* workspace, size_t workspace_bytes, int32_t* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WSVD_B200_H */
