// Declarations shared by the library's translation units (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// Record a message for fa_last_error_string() (thread-local) and return `code`.
int set_error(int code, const char* fmt, ...);

// Device pointer of the per-device error word that kernels set on a bounded
// wait running out or on an out-of-range index read from device memory.
int* device_error_word(int device);

// Encodes a tiled TMA tensor map over 16-bit elements (bf16 or fp16) with
// 128-byte swizzle and zero fill.  dims[0] is the contiguous dimension;
// strides_bytes[i] is the byte stride of dimension i + 1.  Returns an FA_* status.
int encode_tensor_map_16bit(CUtensorMap* m, const void* base, bool bf16, int rank,
                            const uint64_t* dims, const uint64_t* strides_bytes,
                            const uint32_t* box);

// The same over one-byte elements (E4M3 codes).
int encode_tensor_map_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                         const uint64_t* strides_bytes, const uint32_t* box);

// Number of SMs of `device` (cached per device), 0 if it cannot be read.
int device_sm_count(int device);

// Generation of the per-device host caches that depend on the device's context
// (device addresses of the library's __device__ symbols, kernel attributes).
// Starts at 1; fa_release() moves it on, so every such cache is rebuilt on its
// next use (needed after cudaDeviceReset, which gives the device a new context).
int cache_generation();

// Wall-time limit of every bounded wait inside a kernel.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Forward prefill launcher (validated arguments).  bf16 selects bf16 inputs,
// otherwise fp16.  Returns an FA_* status.
// Batch layout of a forward call.  cu_q == nullptr: dense [B, H, N, D] tensors.
// Otherwise queries are packed as [total_q, H, D] with per-sequence row offsets
// cu_q ([B + 1], device) and Nq bounds their lengths; keys/values are either
// packed the same way (cu_k, total_k; Nk bounds their lengths) or, with
// block_table != nullptr, held in a page pool [num_pages, 16, Hkv, D] reached
// through block_table [B, max_pages] with seq_lens_k [B] keys per sequence.
struct FwdLayoutArgs {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int total_q = 0, total_k = 0;
  const int* block_table = nullptr;
  const int* seq_lens_k = nullptr;
  int max_pages = 0, num_pages = 0;
};
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
               const FwdLayoutArgs& la, int B, int Hq, int Hkv, int Nq, int Nk, int D,
               float scale, int causal, bool bf16, cudaStream_t stream, int device);

// Split-KV paged decode launcher (validated arguments).
int launch_decode(const void* q, const void* kcache, const void* vcache, const int32_t* block_table,
                  const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                  int page_size, float scale, int max_pages_per_seq, int num_pages,
                  cudaStream_t stream, int device);

// E4M3 quantisation of a bf16 tensor [Z, N, D] (validated arguments): codes
// [Z, N, D], fp32 scales [Z, ceil(N / 128)] (group_rows 128) or [Z] (0), with
// the optional Walsh-Hadamard rotation by `signs` [D].
int launch_quantize_e4m3(const void* x, void* codes, float* scales, int Z, int N, int D,
                         int group_rows, const float* signs, cudaStream_t stream, int device);

// FP8 (E4M3) forward prefill launcher (validated arguments, D = 128).
int launch_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                   const float* k_scale, const float* v_scale, void* o, float* lse, int B,
                   int Hq, int Hkv, int Nq, int Nk, float scale, int causal, cudaStream_t stream,
                   int device);

// Merge of a partial attention result (o_part bf16 [rows, D], lse_part) into an
// fp32 accumulator (o_acc [rows, D], lse_acc; overwritten when `first`), with
// an optional bf16 copy of the merged rows (validated arguments).
int launch_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                          void* o_out, long long rows, int D, int first, cudaStream_t stream,
                          int device);

// Attention backward with recomputation (validated arguments, bf16): delta
// [B * Hq, Nq] fp32 is written (rowsum(dO * O)), then dK, dV and dQ.
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, cudaStream_t stream,
               int device);

// fa_fwd (bf16) from host buffers through caller-owned device buffers, the
// copies of one chunk overlapping the forward of another (validated arguments).
int launch_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                    float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                    float* lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                    int causal, cudaStream_t stream, int device);
void release_host_pipeline_resources();

// One bounded wait that nothing satisfies, given up after limit_us (validated).
int launch_wait_selftest(unsigned limit_us, int* gave_up, cudaStream_t stream, int device);

// Release cached per-device resources owned by the decode path.
void release_decode_resources();

// Size of the fixed scratch array used by fa_decode_paged_noalloc.
constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB

// Host-side check that a problem fits the fixed scratch of
// fa_decode_paged_noalloc on a device with `nsm` SMs; nsm = 0 checks the
// smallest need of any schedule, without a device.  Returns an FA_* status.
int check_decode_noalloc(int B, int Hq, int Hkv, int max_pages_per_seq, int nsm);

// Split-KV paged decode whose partials live in the library's fixed scratch
// array; allocates nothing.  `device` must be the current device.
int launch_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                          const int32_t* block_table, const int32_t* seq_lens, void* o, float* lse,
                          int B, int Hq, int Hkv, int max_pages_per_seq, int num_pages,
                          float scale, cudaStream_t stream, int device);

}  // namespace fa
