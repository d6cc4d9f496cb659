// C-ABI entry points: argument validation on the host, error reporting and the
// per-device error word.  Every compute step runs in the kernels of
// fa_fwd_sm100.cu and fa_decode_sm100.cu; there is no host fallback.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {

namespace {
thread_local char g_msg[512] = "";
__device__ int g_error_word;   // see kErrTimeout / kErrBadIndex
std::mutex g_err_mu;
int* g_err_ptr[64] = {};
int g_err_gen[64] = {};
std::atomic<int> g_cache_gen{1};
}  // namespace

int cache_generation() { return g_cache_gen.load(std::memory_order_acquire); }

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int* device_error_word(int device) {
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> g(g_err_mu);
  const int gen = cache_generation();
  if (!g_err_ptr[device] || g_err_gen[device] != gen) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[device] = static_cast<int*>(p);
    g_err_gen[device] = gen;
  }
  return g_err_ptr[device];
}

int device_sm_count(int device) {
  static int cached[64] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (device < 0 || device >= 64) return 0;
  if (!cached[device]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) n = 0;
    cached[device] = n;
  }
  return cached[device];
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, reached through the runtime so that loading this
// library needs no driver library at link time.
EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}
}  // namespace

namespace {
int encode_tensor_map(CUtensorMap* m, CUtensorMapDataType type, const void* base, int rank,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = enc(m, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, bx,
                   es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
  return FA_OK;
}
}  // namespace

int encode_tensor_map_16bit(CUtensorMap* m, const void* base, bool bf16, int rank,
                            const uint64_t* dims, const uint64_t* strides_bytes,
                            const uint32_t* box) {
  return encode_tensor_map(
      m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, rank,
      dims, strides_bytes, box);
}

int encode_tensor_map_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                         const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes,
                           box);
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The current device must be an sm_100 part; its ordinal is returned in *dev.
int current_sm100(int* dev) {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return set_error(FA_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  }
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, d);
  if (major != 10 || minor != 0)
    return set_error(FA_ERR_NO_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a",
                     d, major, minor);
  *dev = d;
  return FA_OK;
}

int validate_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv,
                 int Nq, int Nk, int D, float scale, int causal) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dimension %d is not supported (64 or 128)", D);
  if (B == 0 || Hq == 0 || Nq == 0) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  if (causal && Nq > Nk)
    return set_error(FA_ERR_INVALID_ARG, "causal attention needs Nq <= Nk (got %d > %d)", Nq, Nk);
  if (!q || !o || (Nk > 0 && (!k || !v))) return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(o) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return set_error(FA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL || static_cast<long long>(B) * Hkv > 0x7fffffffLL)
    return set_error(FA_ERR_UNSUPPORTED, "B * H too large");
  return FA_OK;
}

int fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, cudaStream_t stream,
               bool bf16) {
  int rc = validate_fwd(q, k, v, o, B, Hq, Hkv, Nq, Nk, D, scale, causal);
  if (rc != FA_OK) return rc;
  if (B == 0 || Hq == 0 || Nq == 0) return FA_OK;
  int dev;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_fwd(q, k, v, o, lse, FwdLayoutArgs{}, B, Hq, Hkv, Nq, Nk, D, scale, causal, bf16,
                    stream, dev);
}

int varlen_common(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_q, const int32_t* cu_k, int B, int Hq, int Hkv,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int D, float scale,
                  int causal, cudaStream_t stream, bool bf16) {
  if (B < 0 || Hq < 0 || Hkv < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || total_q < 0 ||
      total_k < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
  if (B == 0 || Hq == 0 || total_q == 0 || max_seqlen_q == 0) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  if (!q || !o || !cu_q || !cu_k || (total_k > 0 && (!k || !v)))
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(o) || (total_k > 0 && (!aligned16(k) || !aligned16(v))))
    return set_error(FA_ERR_INVALID_ARG, "q, k, v and o must be 16-byte aligned");
  if (static_cast<long long>(total_q) * Hq > 0x7fffffffLL ||
      static_cast<long long>(max_seqlen_q) + 256 > 0x7fffffffLL)
    return set_error(FA_ERR_INVALID_ARG, "total_q * Hq too large");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  FwdLayoutArgs la;
  la.cu_q = cu_q;
  la.cu_k = cu_k;
  la.total_q = total_q;
  la.total_k = total_k;
  return launch_fwd(q, k, v, o, lse, la, B, Hq, Hkv, max_seqlen_q, max_seqlen_k, D, scale, causal,
                    bf16, stream, dev);
}

int paged_common(const void* q, const void* kcache, const void* vcache,
                 const int32_t* block_table, void* o, float* lse, const int32_t* cu_q,
                 const int32_t* seq_lens_k, int B, int Hq, int Hkv, int max_seqlen_q,
                 int max_pages_per_seq, int num_pages, int total_q, int D, int page_size,
                 float scale, int causal, cudaStream_t stream, bool bf16) {
  if (B < 0 || Hq < 0 || Hkv < 0 || max_seqlen_q < 0 || max_pages_per_seq < 0 ||
      num_pages < 0 || total_q < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
  if (page_size != 16)
    return set_error(FA_ERR_UNSUPPORTED, "paged prefill supports page_size == 16 only (got %d)",
                     page_size);
  if (B == 0 || Hq == 0 || total_q == 0 || max_seqlen_q == 0) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  if (max_pages_per_seq <= 0 || num_pages <= 0)
    return set_error(FA_ERR_INVALID_ARG, "max_pages_per_seq and num_pages must be positive");
  if (!q || !kcache || !vcache || !block_table || !o || !cu_q || !seq_lens_k)
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o))
    return set_error(FA_ERR_INVALID_ARG, "q, caches and o must be 16-byte aligned");
  if (static_cast<long long>(max_pages_per_seq) * 16 > 0x7fffffffLL ||
      static_cast<long long>(num_pages) * 16 > 0x7fffffffLL ||
      static_cast<long long>(total_q) * Hq > 0x7fffffffLL)
    return set_error(FA_ERR_INVALID_ARG, "sizes too large");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  FwdLayoutArgs la;
  la.cu_q = cu_q;
  la.total_q = total_q;
  la.block_table = block_table;
  la.seq_lens_k = seq_lens_k;
  la.max_pages = max_pages_per_seq;
  la.num_pages = num_pages;
  return launch_fwd(q, kcache, vcache, o, lse, la, B, Hq, Hkv, max_seqlen_q,
                    max_pages_per_seq * 16, D, scale, causal, bf16, stream, dev);
}

int fwd_host_common(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                    float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                    float* lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                    int causal, cudaStream_t stream) {
  int rc = validate_fwd(q_dev, k_dev, v_dev, o_dev, B, Hq, Hkv, Nq, Nk, D, scale, causal);
  if (rc != FA_OK) return rc;
  if (B == 0 || Hq == 0 || Nq == 0) return FA_OK;
  if (!q_host || !o_host || (Nk > 0 && (!k_host || !v_host)))
    return set_error(FA_ERR_INVALID_ARG, "null host pointer");
  if ((lse_host == nullptr) != (lse_dev == nullptr))
    return set_error(FA_ERR_INVALID_ARG, "lse_host and lse_dev must both be given or both NULL");
  int dev;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev,
                         lse_dev, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dev);
}

int quantize_common(const void* x, void* codes, float* scales, int Z, int N, int D,
                    int group_rows, const float* signs, cudaStream_t stream) {
  if (Z < 0 || N < 0) return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
  if (group_rows != 0 && group_rows != 128)
    return set_error(FA_ERR_UNSUPPORTED, "group_rows must be 128 or 0 (got %d)", group_rows);
  if (Z == 0) return FA_OK;
  if (Z > 65535) return set_error(FA_ERR_UNSUPPORTED, "Z (%d) above 65535", Z);
  if (!scales || (N > 0 && (!x || !codes))) return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (N > 0 && (!aligned16(x) || !aligned16(codes)))
    return set_error(FA_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  if (static_cast<long long>(N) * D * Z > (1LL << 40))
    return set_error(FA_ERR_INVALID_ARG, "tensor too large");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_quantize_e4m3(x, codes, scales, Z, N, D, group_rows, signs, stream, dev);
}

int fwd_fp8_common(const void* q8, const void* k8, const void* v8, const float* q_scale,
                   const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, cudaStream_t stream) {
  int rc = validate_fwd(q8, k8, v8, o, B, Hq, Hkv, Nq, Nk, D, scale, causal);
  if (rc != FA_OK) return rc;
  if (D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "the FP8 forward supports D == 128 only (got %d)", D);
  if (B == 0 || Hq == 0 || Nq == 0) return FA_OK;
  if (!q_scale || (Nk > 0 && (!k_scale || !v_scale)))
    return set_error(FA_ERR_INVALID_ARG, "null scale pointer");
  int dev;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, scale,
                        causal, stream, dev);
}

int merge_common(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                 void* o_out, long long rows, int D, int first, cudaStream_t stream) {
  if (rows < 0) return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
  if (rows == 0) return FA_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part)
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(o_acc) || !aligned16(o_part) || (o_out && !aligned16(o_out)))
    return set_error(FA_ERR_INVALID_ARG, "o_acc, o_part and o_out must be 16-byte aligned");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_merge_partials(o_acc, lse_acc, o_part, lse_part, o_out, rows, D, first ? 1 : 0,
                               stream, dev);
}

int bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, cudaStream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 64 && D != 128)
    return set_error(FA_ERR_UNSUPPORTED, "head dimension %d is not supported (64 or 128)", D);
  if (B == 0 || Hq == 0 || (Nq == 0 && Nk == 0)) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  if (causal && Nq > Nk)
    return set_error(FA_ERR_INVALID_ARG, "causal attention needs Nq <= Nk (got %d > %d)", Nq, Nk);
  const bool has_q = Nq > 0, has_k = Nk > 0;
  if ((has_q && (!q || !o || !lse || !dout || !dq || !delta)) ||
      (has_k && (!k || !v || !dk || !dv)))
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if ((has_q && (!aligned16(q) || !aligned16(o) || !aligned16(dout) || !aligned16(dq))) ||
      (has_k && (!aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv))))
    return set_error(FA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return set_error(FA_ERR_UNSUPPORTED, "B * H too large");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_bwd(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale,
                    causal, stream, dev);
}

}  // namespace
}  // namespace fa

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int Hq, int Hkv,
           int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream) {
  return fa::bwd_common(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale,
                        causal, reinterpret_cast<cudaStream_t>(stream));
}

int fa_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                      void* o_out, long long rows, int D, int first, fa_stream_t stream) {
  return fa::merge_common(o_acc, lse_acc, o_part, lse_part, o_out, rows, D, first,
                          reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                float* lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                int causal, fa_stream_t stream) {
  return fa::fwd_host_common(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev,
                             lse_dev, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                             reinterpret_cast<cudaStream_t>(stream));
}

int fa_quantize_e4m3(const void* x, void* codes, float* scales, int Z, int N, int D,
                     int group_rows, const float* signs, fa_stream_t stream) {
  return fa::quantize_common(x, codes, scales, Z, N, D, group_rows, signs,
                             reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
               const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream) {
  return fa::fwd_fp8_common(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, D,
                            scale, causal, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream) {
  return fa::fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                        reinterpret_cast<cudaStream_t>(stream), true);
}

int fa_fwd_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, fa_stream_t stream) {
  return fa::fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                        reinterpret_cast<cudaStream_t>(stream), false);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                  int Hkv, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int D,
                  float scale, int causal, fa_stream_t stream) {
  return fa::varlen_common(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, max_seqlen_q,
                           max_seqlen_k, total_q, total_k, D, scale, causal,
                           reinterpret_cast<cudaStream_t>(stream), true);
}

int fa_fwd_varlen_fp16(const void* q, const void* k, const void* v, void* o, float* lse,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                       int Hkv, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                       int D, float scale, int causal, fa_stream_t stream) {
  return fa::varlen_common(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, max_seqlen_q,
                           max_seqlen_k, total_q, total_k, D, scale, causal,
                           reinterpret_cast<cudaStream_t>(stream), false);
}

int fa_fwd_paged(const void* q, const void* kcache, const void* vcache,
                 const int32_t* block_table, void* o, float* lse, const int32_t* cu_seqlens_q,
                 const int32_t* seq_lens_k, int B, int Hq, int Hkv, int max_seqlen_q,
                 int max_pages_per_seq, int num_pages, int total_q, int D, int page_size,
                 float scale, int causal, fa_stream_t stream) {
  return fa::paged_common(q, kcache, vcache, block_table, o, lse, cu_seqlens_q, seq_lens_k, B, Hq,
                          Hkv, max_seqlen_q, max_pages_per_seq, num_pages, total_q, D, page_size,
                          scale, causal, reinterpret_cast<cudaStream_t>(stream), true);
}

int fa_decode_paged(const void* q, const void* kcache, const void* vcache,
                    const int32_t* block_table, const int32_t* seq_lens, void* o, int B, int Hq,
                    int Hkv, int D, int page_size, float scale, fa_stream_t stream,
                    int max_pages_per_seq, int num_pages, float* lse) {
  using namespace fa;
  if (B < 0 || Hq < 0 || Hkv < 0 || max_pages_per_seq < 0 || num_pages < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 128) return set_error(FA_ERR_UNSUPPORTED, "decode supports D == 128 only (got %d)", D);
  if (page_size != 16)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports page_size == 16 only (got %d)",
                     page_size);
  if (B == 0 || Hq == 0) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} (got %d)", G);
  if (max_pages_per_seq <= 0 || num_pages <= 0)
    return set_error(FA_ERR_INVALID_ARG, "max_pages_per_seq and num_pages must be positive");
  if (!q || !kcache || !vcache || !block_table || !seq_lens || !o)
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o))
    return set_error(FA_ERR_INVALID_ARG, "q, caches and o must be 16-byte aligned");
  if (static_cast<long long>(max_pages_per_seq) * 16 > 0x7fffffffLL)
    return set_error(FA_ERR_INVALID_ARG, "max_pages_per_seq too large");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_decode(q, kcache, vcache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                       scale, max_pages_per_seq, num_pages, reinterpret_cast<cudaStream_t>(stream),
                       dev);
}

int fa_decode_paged_noalloc(const void* q, const void* kcache, const void* vcache,
                            const int32_t* block_table, const int32_t* seq_lens, void* o, int B,
                            int Hq, int Hkv, int D, int page_size, float scale, fa_stream_t stream,
                            int max_pages_per_seq, int num_pages, float* lse) {
  using namespace fa;
  if (B < 0 || Hq < 0 || Hkv < 0 || max_pages_per_seq < 0 || num_pages < 0)
    return set_error(FA_ERR_INVALID_ARG, "negative size");
  if (!(std::isfinite(scale) && scale > 0.f))
    return set_error(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (D != 128) return set_error(FA_ERR_UNSUPPORTED, "decode supports D == 128 only (got %d)", D);
  if (page_size != 16)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports page_size == 16 only (got %d)",
                     page_size);
  if (B == 0 || Hq == 0) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return set_error(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq,
                     Hkv);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} (got %d)", G);
  if (max_pages_per_seq <= 0 || num_pages <= 0)
    return set_error(FA_ERR_INVALID_ARG, "max_pages_per_seq and num_pages must be positive");
  if (!q || !kcache || !vcache || !block_table || !seq_lens || !o)
    return set_error(FA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o))
    return set_error(FA_ERR_INVALID_ARG, "q, caches and o must be 16-byte aligned");
  if (static_cast<long long>(max_pages_per_seq) * 16 > 0x7fffffffLL)
    return set_error(FA_ERR_INVALID_ARG, "max_pages_per_seq too large");
  int dev, rc;
  // Problems that no schedule fits are rejected before the device is touched;
  // the plan for the device's SM count is checked again at launch.
  if ((rc = check_decode_noalloc(B, Hq, Hkv, max_pages_per_seq, 0)) != FA_OK) return rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_decode_noalloc(q, kcache, vcache, block_table, seq_lens, o, lse, B, Hq, Hkv,
                               max_pages_per_seq, num_pages, scale,
                               reinterpret_cast<cudaStream_t>(stream), dev);
}

int fa_selftest_wait_timeout(unsigned int limit_us, int* gave_up, fa_stream_t stream) {
  using namespace fa;
  if (limit_us == 0 || limit_us > 1000000u)
    return set_error(FA_ERR_INVALID_ARG, "limit_us must be in [1, 1000000] (got %u)", limit_us);
  if (gave_up && (reinterpret_cast<uintptr_t>(gave_up) & 3u))
    return set_error(FA_ERR_INVALID_ARG, "gave_up must be 4-byte aligned");
  int dev, rc;
  if ((rc = current_sm100(&dev)) != FA_OK) return rc;
  return launch_wait_selftest(limit_us, gave_up, reinterpret_cast<cudaStream_t>(stream), dev);
}

const char* fa_last_error_string(void) { return fa::g_msg; }

int fa_device_status(void) {
  using namespace fa;
  int dev;
  int rc = current_sm100(&dev);
  if (rc != FA_OK) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "device: %s", cudaGetErrorString(e));
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int));
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
  if (word == 0) return FA_OK;
  const int zero = 0;
  cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
  if (word & kErrTimeout)
    return set_error(FA_ERR_DEVICE_TIMEOUT, "a bounded in-kernel wait ran out (word 0x%x)", word);
  if (word & kErrDiverged)
    return set_error(FA_ERR_DEVICE_DIVERGED,
                     "a tensor-memory access found its warp diverged (word 0x%x)", word);
  return set_error(FA_ERR_DEVICE_INDEX, "out-of-range block-table entry or length (word 0x%x)",
                   word);
}

void fa_release(void) {
  fa::release_decode_resources();
  fa::release_host_pipeline_resources();
  // cached device addresses and kernel attributes are looked up again on next use
  fa::g_cache_gen.fetch_add(1, std::memory_order_acq_rel);
}

int fa_version(void) { return 100; }

}  // extern "C"
