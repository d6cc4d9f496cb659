/*
 * Exact tiled attention for NVIDIA B200 (sm_100a): C ABI.
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * tile by tile with the online-softmax decomposition (running row maximum and
 * row sum, old partial results rescaled by exp(m_old - m_new)), so the
 * Nq x Nk score matrix never reaches device memory.  Sources:
 *   - unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency":
 *     opening listing standard_attention (the definition), section "The
 *     Mathematics of Flash Attention" (softmax decomposition and merge) and
 *     section "Implementation Details" (the blockwise loop with running M, L).
 *   - devhandbook.co.kr, "Flash Attention 2 ... PyTorch native": example 1
 *     ([B, H, L, D] tensors), example 3 (is_causal), example 5 (GQA, 32 query
 *     heads over 8 KV heads), section 4 (head dimension 64 or 128).
 *   - cabseo.com, "Advanced techniques for enhancing LLM throughput": sections
 *     "Memory requirements" (KV cache), "Autoregressive and memory-bound
 *     operations" (one query token per decode step) and "Paged attention".
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, contiguous row-major.  The library keeps no reference to them
 *     after the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise the device.
 *   - Return value: FA_OK (0) or an FA_ERR_* code; fa_last_error_string()
 *     then describes the failure (per calling thread).  Argument errors are
 *     detected on the host before anything is launched.
 *   - Faults found inside a kernel (a bounded wait that ran out, an out-of-range
 *     block-table entry or sequence length) do not trap: the kernel skips the
 *     bad work and sets a per-device error word that fa_device_status() reads.
 *   - There is no CPU fallback: without a usable sm_100 device the calls fail.
 */
#ifndef EXACT_TILED_ATTENTION_FA_H
#define EXACT_TILED_ATTENTION_FA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* identical to cudaStream_t */

enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, bad scale */
  FA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (head dim, page size, group size) */
  FA_ERR_CUDA = 3,           /* a CUDA runtime call or kernel launch failed */
  FA_ERR_DEVICE_TIMEOUT = 4, /* fa_device_status(): a bounded in-kernel wait ran out */
  FA_ERR_DEVICE_INDEX = 5,   /* fa_device_status(): a block-table entry or length was out of range */
  FA_ERR_NO_DEVICE = 6,      /* no sm_100 device is current */
  FA_ERR_DEVICE_DIVERGED = 7 /* fa_device_status(), FA_DEBUG builds only: a tensor-memory
                                load/store found its warp diverged and was skipped */
};

/*
 * Prefill / full attention, bf16 inputs and output.
 *
 * Computes O = softmax(scale * Q K^T [+ causal]) V and LSE per query row.
 *   q   [B, Hq,  Nq, D] bf16          k, v [B, Hkv, Nk, D] bf16
 *   o   [B, Hq,  Nq, D] bf16 (written)
 *   lse [B, Hq,  Nq]    fp32 (written; may be NULL): natural log of the row
 *       sum of exp(scale * q.k) over the visible keys.
 * GQA: query head h reads KV head h / (Hq / Hkv); Hq must be a multiple of Hkv.
 * causal != 0: query i sees key j iff j <= i + (Nk - Nq) (bottom-right
 *   alignment; query i sees keys 0..i when Nq == Nk); requires Nq <= Nk.
 * D must be 64 or 128.  scale must be finite and > 0 (the pages use 1/sqrt(D)).
 * B, Hq or Nq equal to 0 is a no-op.  Nk == 0 (non-causal) writes O = 0 and
 * LSE = -inf.
 * Device memory touched: exactly q, k, v (read) and o, lse (written); no
 * workspace is allocated.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream);

/* Same as fa_fwd with fp16 q, k, v and o (fp32 LSE). */
int fa_fwd_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream);

/*
 * Prefill over a ragged batch packed without padding (bf16).
 *
 * Sequence b owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]); its queries see only its own keys.
 * This is the padded batch of devhandbook.co.kr "Flash Attention 2 ... PyTorch
 * native", example 3 (causal rule with a padding mask) without the padding, for
 * the length-mixed batches of cabseo.com "Advanced techniques for enhancing LLM
 * throughput", section "Continuous batching".
 *   q   [total_q, Hq,  D] bf16        k, v [total_k, Hkv, D] bf16
 *   o   [total_q, Hq,  D] bf16 (written rows of valid sequences only)
 *   lse [Hq, total_q]     fp32 (written; may be NULL), as for fa_fwd
 *   cu_seqlens_q, cu_seqlens_k  [B + 1] int32 on the device, non-decreasing,
 *       starting at 0 and ending at most at total_q / total_k.
 *   max_seqlen_q, max_seqlen_k  bounds on every sequence's lengths (the grid is
 *       sized from max_seqlen_q).
 * causal: bottom-right aligned within each sequence; needs Nq_b <= Nk_b.
 * GQA, D, scale and the empty cases as for fa_fwd; a sequence with no keys gets
 * O = 0 and LSE = -inf.  The host cannot read the offsets: a sequence whose
 * offsets break these rules (or whose length exceeds the bound) is skipped, its
 * rows are not written, and FA_ERR_DEVICE_INDEX is raised in fa_device_status().
 * No workspace is allocated.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                  int Hkv, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int D,
                  float scale, int causal, fa_stream_t stream);

/* Same as fa_fwd_varlen with fp16 q, k, v and o (fp32 LSE). */
int fa_fwd_varlen_fp16(const void* q, const void* k, const void* v, void* o, float* lse,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                       int Hkv, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                       int D, float scale, int causal, fa_stream_t stream);

/*
 * Prefill against a paged KV cache (bf16): the new query tokens of each
 * sequence attend over that sequence's keys and values held in the page pool
 * (cabseo.com "Advanced techniques for enhancing LLM throughput", section
 * "Paged attention"), e.g. a prompt prefilled in chunks after earlier chunks
 * were written to the cache.
 *   q            [total_q, Hq, D] bf16, sequence b's queries are rows
 *                [cu_seqlens_q[b], cu_seqlens_q[b+1]) (int32 [B + 1] on the device)
 *   kcache/vcache [num_pages, page_size, Hkv, D] bf16, as for fa_decode_paged
 *   block_table  [B, max_pages_per_seq] int32, seq_lens_k [B] int32: sequence b
 *                has seq_lens_k[b] keys, token t in page block_table[b][t / 16]
 *   o            [total_q, Hq, D] bf16 (written rows of valid sequences only)
 *   lse          [Hq, total_q] fp32 (written; may be NULL)
 * causal: the queries are the last Nq_b tokens of the sequence (bottom-right
 * alignment); needs Nq_b <= seq_lens_k[b].  Supported: page_size == 16, D 64 or
 * 128, GQA as for fa_fwd.  Lengths and offsets breaking these rules skip the
 * sequence and raise FA_ERR_DEVICE_INDEX; a block-table entry outside
 * [0, num_pages) is read as page 0 and raises the same status.  No workspace is
 * allocated.
 */
int fa_fwd_paged(const void* q, const void* kcache, const void* vcache,
                 const int32_t* block_table, void* o, float* lse, const int32_t* cu_seqlens_q,
                 const int32_t* seq_lens_k, int B, int Hq, int Hkv, int max_seqlen_q,
                 int max_pages_per_seq, int num_pages, int total_q, int D, int page_size,
                 float scale, int causal, fa_stream_t stream);

/*
 * fa_fwd (bf16) with the inputs in HOST memory and the outputs wanted there.
 *   q_host, k_host, v_host, o_host, lse_host: host buffers with fa_fwd's layouts
 *     (page-locked for the copies to run asynchronously and overlap)
 *   q_dev, k_dev, v_dev, o_dev, lse_dev: device buffers of the same sizes, owned
 *     by the caller, used as staging (their contents are overwritten)
 *   lse_host and lse_dev are both given or both NULL.
 * The work is cut into chunks of whole sequences (B >= 8) or whole GQA groups
 * of a sequence (sized 1:3:3:1 when B >= 8 or B = 1: small first and last
 * chunks); each chunk's inputs are copied in while the previous chunk is
 * computed and the one before it copied out, on two library-owned copy streams
 * ordered against `stream` by events: the call is asynchronous on `stream` like
 * fa_fwd, and the host outputs are complete once `stream` reaches the point of
 * the call.  fa_release() destroys the copy streams.  Argument rules as fa_fwd.
 */
int fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                float* lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                int causal, fa_stream_t stream);

/*
 * E4M3 (FP8) quantisation of a bf16 tensor, the input preparation of
 * fa_fwd_fp8.  unite.ai, "Flash Attention: Revolutionizing Transformer
 * Efficiency", section "Flash Attention-3", names FP8 inputs with block
 * quantisation and incoherent processing without defining them; this entry
 * point takes the plainest reading:
 *   x       [Z, N, D] bf16 (Z slices of N rows, e.g. Z = B * H)
 *   codes   [Z, N, D] uint8 E4M3 codes (written): sign bit 7, exponent bits 3-6
 *           (bias 7), mantissa bits 0-2, largest finite value 448
 *   scales  fp32 (written), x ~= code * scale of the row's group:
 *           group_rows == 128: [Z, ceil(N / 128)], one per 128-row group;
 *           group_rows == 0:   [Z], one per slice.
 *   signs   [D] fp32 of +1.0 / -1.0, or NULL.  When given, every row is first
 *           multiplied by diag(signs) H / sqrt(D) (H the Walsh-Hadamard matrix,
 *           H[i][j] = (-1)^popcount(i & j)): an orthogonal map, applied to Q and
 *           K alike, that leaves Q K^T unchanged and spreads outliers.
 * Per group: amax = max |x| (after the rotation), scale = amax / 448 and
 * r = 448 / amax (both rounded to fp32; 1 when amax == 0), code = E4M3 of the
 * fp32 product x * r, rounded to nearest even, finite values beyond 448
 * saturating.  The rotation runs in fp32 as the fast Walsh-Hadamard transform
 * (butterfly stages in increasing bit order) after one fp32 product per element
 * by sign / sqrt(D).  Supported: D in {64, 128}, group_rows in {128, 0},
 * Z <= 65535.  group_rows == 0 takes three kernel launches and a memset of
 * `scales` on `stream`; no workspace is allocated.  Inputs must be finite.
 */
int fa_quantize_e4m3(const void* x, void* codes, float* scales, int Z, int N, int D,
                     int group_rows, const float* signs, fa_stream_t stream);

/*
 * FP8 (E4M3) prefill: O = softmax(scale * Q K^T [+ causal]) V on quantised
 * inputs (section "Flash Attention-3" of the unite.ai page above: FP8 with
 * block quantisation).
 *   q8  [B, Hq,  Nq, 128] uint8 E4M3 codes, q_scale [B * Hq,  ceil(Nq / 128)] fp32
 *   k8  [B, Hkv, Nk, 128] uint8 E4M3 codes, k_scale [B * Hkv, ceil(Nk / 128)] fp32
 *   v8  [B, Hkv, Nk, 128] uint8 E4M3 codes, v_scale [B * Hkv] fp32
 *   o   [B, Hq, Nq, 128] bf16 (written), lse [B, Hq, Nq] fp32 (written; may be NULL)
 * i.e. exactly what fa_quantize_e4m3 writes for group_rows 128 (q, k) and 0 (v);
 * the inputs represent q8 * q_scale of the row's 128-row group, and so on.
 * Scales must be positive and finite (other values give unspecified numbers,
 * never an out-of-range access).  Causal masking, GQA and the argument rules
 * are those of fa_fwd; D == 128 only.  Q K^T and P V run on the tensor cores
 * in E4M3 with fp32 accumulation; P is rounded to E4M3 before P V (at most
 * 2^-4 relative error per normal entry), the row sums are kept in fp32.
 */
int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
               const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream);

/*
 * Backward pass of fa_fwd (bf16) with recomputation: unite.ai page above, which
 * names recomputation (P is not stored; it is rebuilt tile by tile from the
 * saved LSE).  With P = exp(scale Q K^T - LSE) (causal: bottom-right mask) and
 * delta_i = sum_d dO_id O_id:
 *     dV = P^T dO,  dS = P * (dO V^T - delta),  dQ = scale dS K,  dK = scale dS^T Q;
 * the query heads of a KV head add into its dK and dV (GQA).
 *   q, o, dout [B, Hq, Nq, D] bf16; k, v [B, Hkv, Nk, D] bf16
 *   lse        [B, Hq, Nq] fp32 (fa_fwd's LSE for the same inputs)
 *   dq         [B, Hq, Nq, D] bf16 (written); dk, dv [B, Hkv, Nk, D] bf16 (written)
 *   delta      [B, Hq, Nq] fp32 (written: rowsum(dout * o), caller-provided scratch)
 * Rules of fa_fwd for sizes, GQA, causal and alignment; D in {64, 128}.  Keys
 * that no query sees get dK = dV = 0.  Three kernels, no atomics, nothing
 * allocated: rows of delta, then dK/dV (a CTA per key tile), then dQ (a CTA per
 * query tile); P and dS are rounded to bf16 before their tensor-core products.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int Hq, int Hkv,
           int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream);

/*
 * Self-test of the bounded in-kernel waits (failure detection without a fault).
 * Launches one thread that waits on a barrier nothing ever completes; after
 * limit_us microseconds (1 .. 1000000) the wait gives up, sets the timeout bit
 * of the device error word and the kernel returns.  The next fa_device_status()
 * then reports FA_ERR_DEVICE_TIMEOUT (and clears the word); the context stays
 * usable.  gave_up (device int, may be NULL) receives 1 if the wait gave up,
 * 0 if it was satisfied.  Every other kernel of the library waits through the
 * same routine, with a limit of 2 s.
 */
int fa_selftest_wait_timeout(unsigned int limit_us, int* gave_up, fa_stream_t stream);

/*
 * Merge of partial attention results over disjoint key sets (the combine step
 * of the split-KV decode, exposed for sequence-sharded prefill: each rank's
 * queries meet the K/V chunks of every rank and fold each chunk's result in).
 * unite.ai page above, section "The Mathematics of Flash Attention": with
 * normalised partial outputs and their log-sum-exps,
 *     lse = log(e^lse_acc + e^lse_part),
 *     O   = e^(lse_acc - lse) O_acc + e^(lse_part - lse) O_part.
 *   o_acc    [rows, D] fp32, read (unless `first`) and written
 *   lse_acc  [rows] fp32, read (unless `first`) and written; -inf = no key yet
 *   o_part   [rows, D] bf16 (e.g. fa_fwd's output over one key chunk)
 *   lse_part [rows] fp32 (fa_fwd's LSE over that chunk; -inf = no key)
 *   o_out    [rows, D] bf16, written with the merged rows when not NULL
 *   first    nonzero: the accumulator is set to the part (o_acc, lse_acc not read)
 * Rows where both LSEs are -inf get O = 0, LSE = -inf.  D in {64, 128}.
 */
int fa_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                      void* o_out, long long rows, int D, int first, fa_stream_t stream);

/*
 * Decode over a paged KV cache: one new query token per sequence attends over
 * all of that sequence's cached keys and values (no mask beyond its length).
 *   q           [B, Hq, D] bf16
 *   kcache      [num_pages, page_size, Hkv, D] bf16  (token slot t of a page
 *   vcache      [num_pages, page_size, Hkv, D] bf16   holds all Hkv heads)
 *   block_table [B, max_pages_per_seq] int32: page ids of sequence b in token
 *               order; token t lives in page block_table[b][t / page_size],
 *               slot t % page_size.  Entries past the sequence are not read.
 *   seq_lens    [B] int32, 0 <= seq_lens[b] <= max_pages_per_seq * page_size
 *   o           [B, Hq, D] bf16 (written)
 *   lse         [B, Hq] fp32 (written; may be NULL)
 * Supported: D == 128, page_size == 16, Hq / Hkv in {1, 2, 4, 8}.
 * num_pages bounds every block-table entry (0 <= id < num_pages); entries out
 * of range are skipped and flagged in the device error word.
 * A sequence of length 0 gets O = 0 and LSE = -inf.
 * Work is split over key chunks; partial results are merged by their LSE.
 * For Hkv <= 8 one persistent CTA per SM takes an equal share of all
 * sequences' cache (so ragged lengths stay balanced); otherwise the grid is
 * (chunk, sequence).  The partials live in a stream-ordered workspace taken
 * from a library-owned memory pool on `stream` and returned to it on `stream`
 * (no device sync); fa_release() frees the pool.
 */
int fa_decode_paged(const void* q, const void* kcache, const void* vcache,
                    const int32_t* block_table, const int32_t* seq_lens, void* o, int B, int Hq,
                    int Hkv, int D, int page_size, float scale, fa_stream_t stream,
                    int max_pages_per_seq, int num_pages, float* lse);

/*
 * fa_decode_paged without any device-memory allocation.
 *
 * The pages have no counterpart of this entry point; it exists for callers that
 * cannot allocate device memory while they decode.  A serving engine typically
 * reserves nearly all device memory up front (weights, the KV-cache page pool)
 * and must not have a decode step fail or stall on an allocation; some
 * runtimes forbid driver allocations after start-up altogether.
 * fa_decode_paged takes its chunk workspace from a memory pool on every call;
 * this variant instead keeps the chunk partials in a fixed 16 MiB array that is
 * compiled into the library, so it calls no cudaMalloc, cudaFree or pool
 * allocation.
 *
 * Arguments, layouts, supported sizes, outputs and error codes are those of
 * fa_decode_paged.  Differences:
 *   - The partial results are rows of 516 bytes (128 fp32 values and an LSE).
 *     With Hkv <= 8 (any supported Hq/Hkv) the persistent schedule needs
 *     (C + B) * Hq of them plus (B + 2) * 4 bytes of offsets, C being the
 *     device's SM count: it fits when (C + B) * Hq * 516 + (B + 2) * 4 <=
 *     16 MiB (C = 148, Hq = 32: B <= 867).
 *     Problems that it does not fit, and every problem with Hkv > 8, use the
 *     (chunk, sequence) schedule with B * Hq * chunks rows, the chunks being
 *     widened until they fit (then the result agrees with fa_decode_paged
 *     within rounding, not bit for bit).  A problem with B * Hq > 32,513
 *     (B * Hq * 516 > 16 MiB) fits neither and is rejected with
 *     FA_ERR_INVALID_ARG before anything touches the device.
 *   - The array is shared by every call and keeps the previous call's contents
 *     (nothing in it needs to start at zero).  Calls whose kernels overlap on
 *     the GPU, e.g. issued on two streams without ordering, race on it.
 *   - The 16 MiB are held on every GPU on which the library's kernels are
 *     loaded, until the process exits.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.  After cudaDeviceReset the looked-up address is stale:
 *     call fa_release() before the next call, which makes it look it up again.
 */
int fa_decode_paged_noalloc(const void* q, const void* kcache, const void* vcache,
                            const int32_t* block_table, const int32_t* seq_lens, void* o, int B,
                            int Hq, int Hkv, int D, int page_size, float scale,
                            fa_stream_t stream, int max_pages_per_seq, int num_pages, float* lse);

/* Description of the last error returned on this thread ("" if none). */
const char* fa_last_error_string(void);

/*
 * Synchronises the current device, then reads and clears its device error
 * word.  Returns FA_OK, FA_ERR_DEVICE_TIMEOUT, FA_ERR_DEVICE_INDEX,
 * FA_ERR_DEVICE_DIVERGED (FA_DEBUG builds) or FA_ERR_CUDA; when several bits
 * are set the first of timeout, divergence, index is reported.
 */
int fa_device_status(void);

/*
 * Frees the library's cached device resources (decode workspace pools, the host
 * pipeline's streams) and forgets every cached per-device lookup
 * (device addresses of the library's symbols, kernel attributes), which are
 * redone on the next call.  Call it after cudaDeviceReset and before using the
 * library again on that device.  No call of the library may run concurrently.
 */
void fa_release(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_FA_H */
