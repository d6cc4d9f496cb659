// Forward from host buffers: fa_fwd with the inputs in host memory and the
// outputs wanted back there.
//
// The work is cut into chunks of whole sequences (B >= 8), of whole GQA groups
// of the one sequence (B = 1), both in the proportions 1:3:3:1, or of about
// 8 / B group ranges per sequence otherwise; each chunk is contiguous in every
// tensor.  Chunk c's inputs are copied in on a copy
// stream while chunk c - 1 is computed on the caller's stream and chunk c - 2's
// outputs are copied out on a second copy stream, so the host-to-device and
// device-to-host transfers (separate directions of the link) overlap each
// other and the kernels.  Events order the three streams; the call is ordered
// after earlier work on the caller's stream and before later work on it, and
// never synchronises the host.  Every forward is the library's own kernel on
// the chunk's slice of the caller's device buffers.
#include <algorithm>
#include <mutex>
#include <vector>

#include "fa_internal.h"
#include "../../include/fa.h"

namespace fa {
namespace {

struct CopyStreams {
  cudaStream_t in = nullptr;
  cudaStream_t out = nullptr;
};
std::mutex g_cs_mu;
CopyStreams g_cs[64];

int copy_streams(int device, CopyStreams* cs) {
  if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> g(g_cs_mu);
  CopyStreams& s = g_cs[device];
  if (!s.in) {
    cudaError_t e = cudaStreamCreateWithFlags(&s.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s.out, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
      s.in = s.out = nullptr;
      return set_error(FA_ERR_CUDA, "cudaStreamCreateWithFlags: %s", cudaGetErrorString(e));
    }
  }
  *cs = s;
  return FA_OK;
}

struct Chunk {
  int b0, nb;   // sequences
  int g0, ng;   // KV-head groups of each (all of them when nb > 1)
};

// Sizes of the chunks of n units in the proportions 1:3:3:1: a small first
// chunk lets the kernels start early and a small last chunk leaves little to
// copy out after the last kernel, while the middle chunks keep both copy
// directions busy (B1 Hq32 Hkv8 N8192 D128 causal prefill on a B200: 2.69 ms
// per call against 2.87 ms with eight equal chunks and 2.76 ms with four).
std::vector<int> chunk_sizes(int n) {
  if (n < 4) return std::vector<int>(n, 1);
  const int edge = std::max(1, n / 8);
  const int mid = n - 2 * edge;
  return {edge, (mid + 1) / 2, mid / 2, edge};
}

std::vector<Chunk> plan_chunks(int B, int Hkv) {
  std::vector<Chunk> out;
  if (B >= 8) {                       // chunks of whole sequences
    int b0 = 0;
    for (int n : chunk_sizes(B)) {
      out.push_back({b0, n, 0, Hkv});
      b0 += n;
    }
  } else if (B == 1) {                // chunks of whole GQA groups of the sequence
    int g0 = 0;
    for (int n : chunk_sizes(Hkv)) {
      out.push_back({0, 1, g0, n});
      g0 += n;
    }
  } else {                            // each sequence in about 8 / B group chunks
    constexpr int kTarget = 8;
    const int parts = std::min(Hkv, (kTarget + B - 1) / B);
    const int per = (Hkv + parts - 1) / parts;
    for (int b = 0; b < B; ++b)
      for (int g0 = 0; g0 < Hkv; g0 += per) out.push_back({b, 1, g0, std::min(per, Hkv - g0)});
  }
  return out;
}

}  // namespace

int launch_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                    float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                    float* lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int D, float scale,
                    int causal, cudaStream_t stream, int device) {
  CopyStreams cs;
  int rc = copy_streams(device, &cs);
  if (rc != FA_OK) return rc;
  const std::vector<Chunk> chunks = plan_chunks(B, Hkv);
  const int G = Hq / Hkv;
  const size_t q_head = static_cast<size_t>(Nq) * D * 2;    // bytes of one head of q / o
  const size_t kv_head = static_cast<size_t>(Nk) * D * 2;   // bytes of one head of k / v
  const size_t lse_head = static_cast<size_t>(Nq) * 4;
  auto at = [](const void* p, size_t off) {
    return static_cast<const void*>(static_cast<const char*>(p) + off);
  };
  auto at_mut = [](void* p, size_t off) { return static_cast<void*>(static_cast<char*>(p) + off); };

  std::vector<cudaEvent_t> evs;
  auto event = [&](cudaEvent_t* e) {
    cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r == cudaSuccess) evs.push_back(*e);
    return r;
  };
  auto fail = [&](cudaError_t e, const char* what) {
    for (cudaEvent_t x : evs) cudaEventDestroy(x);   // released once their work completes
    return set_error(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  };
  cudaEvent_t start, end;
  cudaError_t e = event(&start);
  if (e != cudaSuccess) return fail(e, "cudaEventCreate");
  // the device buffers may still be in use by earlier work on the caller's stream
  if ((e = cudaEventRecord(start, stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs.in, start, 0)) != cudaSuccess)
    return fail(e, "stream ordering");
  for (const Chunk& c : chunks) {
    const int qh0 = c.b0 * Hq + c.g0 * G;      // first query head (over B * Hq)
    const int nqh = c.nb * c.ng * G;
    const int kh0 = c.b0 * Hkv + c.g0;         // first KV head (over B * Hkv)
    const int nkh = c.nb * c.ng;
    cudaEvent_t in, done;
    if ((e = event(&in)) != cudaSuccess || (e = event(&done)) != cudaSuccess)
      return fail(e, "cudaEventCreate");
    const size_t qo = qh0 * q_head, ko = kh0 * kv_head;
    if ((e = cudaMemcpyAsync(at_mut(q_dev, qo), at(q_host, qo), nqh * q_head,
                             cudaMemcpyHostToDevice, cs.in)) != cudaSuccess ||
        (Nk > 0 && (e = cudaMemcpyAsync(at_mut(k_dev, ko), at(k_host, ko), nkh * kv_head,
                                        cudaMemcpyHostToDevice, cs.in)) != cudaSuccess) ||
        (Nk > 0 && (e = cudaMemcpyAsync(at_mut(v_dev, ko), at(v_host, ko), nkh * kv_head,
                                        cudaMemcpyHostToDevice, cs.in)) != cudaSuccess) ||
        (e = cudaEventRecord(in, cs.in)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(stream, in, 0)) != cudaSuccess)
      return fail(e, "copy in");
    float* lse_c = lse_dev ? lse_dev + static_cast<size_t>(qh0) * Nq : nullptr;
    rc = launch_fwd(at(q_dev, qo), Nk > 0 ? at(k_dev, ko) : nullptr,
                    Nk > 0 ? at(v_dev, ko) : nullptr, at_mut(o_dev, qo), lse_c, FwdLayoutArgs{},
                    c.nb, c.nb > 1 ? Hq : c.ng * G, c.nb > 1 ? Hkv : c.ng, Nq, Nk, D, scale,
                    causal, true, stream, device);
    if (rc != FA_OK) {
      for (cudaEvent_t x : evs) cudaEventDestroy(x);
      return rc;
    }
    if ((e = cudaEventRecord(done, stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(cs.out, done, 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(at_mut(o_host, qo), at(o_dev, qo), nqh * q_head,
                             cudaMemcpyDeviceToHost, cs.out)) != cudaSuccess ||
        (lse_host && (e = cudaMemcpyAsync(lse_host + static_cast<size_t>(qh0) * Nq, lse_c,
                                          nqh * lse_head, cudaMemcpyDeviceToHost, cs.out)) !=
                         cudaSuccess))
      return fail(e, "copy out");
  }
  if ((e = event(&end)) != cudaSuccess) return fail(e, "cudaEventCreate");
  if ((e = cudaEventRecord(end, cs.out)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(stream, end, 0)) != cudaSuccess)
    return fail(e, "stream ordering");
  for (cudaEvent_t x : evs) cudaEventDestroy(x);       // released once their work completes
  return FA_OK;
}

void release_host_pipeline_resources() {
  std::lock_guard<std::mutex> g(g_cs_mu);
  for (auto& s : g_cs) {
    if (s.in) cudaStreamDestroy(s.in);
    if (s.out) cudaStreamDestroy(s.out);
    s.in = s.out = nullptr;
  }
}

}  // namespace fa
