// Split-KV decode over a paged KV cache for sm_100a.
//
// Decode (cabseo.com, "Advanced techniques for enhancing LLM throughput",
// sections "Memory requirements" and "Autoregressive and memory-bound
// operations") attends one new query token per sequence over the whole KV
// cache, a matrix-vector product bound by HBM bandwidth.  The cache is paged
// (section "Paged attention"): fixed pages of 16 token slots, each slot holding
// all KV heads, reached through a per-sequence block table.
//
// Kernel 1 (split): grid (split, sequence).  A CTA streams the pages
// [split * pps, (split + 1) * pps) of one sequence; warp w handles KV head w (and
// w + 8, ...) together with the Hq/Hkv query heads that share it, so every cache
// byte is read from HBM exactly once.  Within a warp each half-warp takes one
// token and each of its 16 lanes a 16-byte slice (8 elements) of the 256-byte
// head row, so a token row is one coalesced 256-byte read.  Partial dot products
// for the G query heads are folded across the 16 lanes with a transposing
// butterfly (each exchange halves the number of live heads), leaving every lane
// with the full score of one head.  An online softmax (running max, rescale by
// exp2(m_old - m_new), unnormalised accumulator) runs over the chunk, and the
// chunk's normalised output and LSE go to a workspace.
// Kernel 2 (combine): merges a sequence's chunks by their LSE -- the softmax
// merge of unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency",
// section "The Mathematics of Flash Attention", formula 2.
#include <cstdio>
#include <mutex>
#include <vector>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {
namespace {

constexpr int kDecD = 128;
constexpr int kPage = 16;
constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994530942f;

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int32_t* block_table;
  const int32_t* seq_lens;
  uint16_t* o;
  float* lse;
  float* ws_o;     // [B][nsplit][Hq][128] normalised chunk outputs
  float* ws_lse;   // [B][nsplit][Hq] chunk LSE (natural log)
  int B, Hq, Hkv, max_pages, num_pages, pps, nsplit;
  float scale_log2;
  int* err;
};

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ int checked_len(const DecodeParams& p, int b) {
  const int len = p.seq_lens[b];
  if (len < 0 || len > p.max_pages * kPage) return -1;
  return len;
}

// Fold G partial sums held by 16 lanes (lane bits 0-3 = sub) into one full sum
// per lane: lane `sub` ends with the total of head sub >> (4 - log2 G).
template <int G>
__device__ __forceinline__ float fold_heads(float (&v)[G], int sub) {
  constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
#pragma unroll
  for (int step = 0; step < LG; ++step) {
    const int mask = 8 >> step;
    const bool upper = (sub & mask) != 0;
    const int n = G >> (step + 1);
#pragma unroll
    for (int k = 0; k < n; ++k) {
      const float keep = upper ? v[k + n] : v[k];
      const float send = upper ? v[k] : v[k + n];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  }
  float x = v[0];
#pragma unroll
  for (int mask = 8 >> LG; mask >= 1; mask >>= 1) x += __shfl_xor_sync(0xffffffffu, x, mask);
  return x;
}

template <int G>
__global__ void __launch_bounds__(kDecThreads) fa_decode_split_kernel(const DecodeParams p) {
  constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  constexpr int SHIFT = 4 - LG;       // lane `h << SHIFT` holds head h after the fold
  constexpr int NI = G >= 8 ? 4 : 8;  // token pairs per iteration
  __shared__ __align__(16) float pbuf[kDecWarps][NI][2][G];

  const int b = blockIdx.y;
  const int split = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int sub = lane & 15;
  const int my_head = sub >> SHIFT;

  const int len = checked_len(p, b);
  if (len < 0) {
    if (threadIdx.x == 0 && split == 0) atomicOr(p.err, kErrBadIndex);
    return;
  }
  const int npages = (len + kPage - 1) / kPage;
  const int pbeg = split * p.pps;
  if (pbeg >= npages) return;
  const int pend = min(pbeg + p.pps, npages);
  const size_t tok_stride = static_cast<size_t>(p.Hkv) * kDecD;   // elements between slots

  for (int g = warp; g < p.Hkv; g += kDecWarps) {
    const int hq0 = g * G;
    float qf[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint4 u = *reinterpret_cast<const uint4*>(
          p.q + (static_cast<size_t>(b) * p.Hq + hq0 + h) * kDecD + sub * 8);
      bf16x8_to_f32(u, qf[h]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[h][e] *= p.scale_log2;
    }
    float m[G], l[G], acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
    }
    float m_mine = -INFINITY;

    for (int pg = pbeg; pg < pend; ++pg) {
      const int page = p.block_table[static_cast<size_t>(b) * p.max_pages + pg];
      if (page < 0 || page >= p.num_pages) {
        if (lane == 0) atomicOr(p.err, kErrBadIndex);
        continue;
      }
      const int ntok = min(kPage, len - pg * kPage);
      const uint16_t* kbase = p.kc + (static_cast<size_t>(page) * kPage * p.Hkv + g) * kDecD + sub * 8;
      const uint16_t* vbase = p.vc + (static_cast<size_t>(page) * kPage * p.Hkv + g) * kDecD + sub * 8;
#pragma unroll 1
      for (int t0 = 0; t0 < kPage; t0 += 2 * NI) {
        uint4 kr[NI], vr[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          const int t = t0 + 2 * i + half;
          if (t < ntok) {
            kr[i] = ld_stream(kbase + t * tok_stride);
            vr[i] = ld_stream(vbase + t * tok_stride);
          } else {
            kr[i] = make_uint4(0, 0, 0, 0);
            vr[i] = make_uint4(0, 0, 0, 0);
          }
        }
        float sc[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          float kf[8];
          bf16x8_to_f32(kr[i], kf);
          float part[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) a = fmaf(qf[h][e], kf[e], a);
            part[h] = a;
          }
          sc[i] = fold_heads<G>(part, sub);
          if (t0 + 2 * i + half >= ntok) sc[i] = -INFINITY;
        }
        // chunk maximum of this lane's head over both half-warps' tokens
        float mx = sc[0];
#pragma unroll
        for (int i = 1; i < NI; ++i) mx = fmaxf(mx, sc[i]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new_mine = fmaxf(m_mine, mx);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mh = fmaxf(m[h], __shfl_sync(0xffffffffu, mx, h << SHIFT));
          const float alpha = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mh);
          l[h] *= alpha;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[h][e] *= alpha;
          m[h] = mh;
        }
        m_mine = m_new_mine;
        float pv[NI];
        float psum = 0.f;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          pv[i] = (sc[i] == -INFINITY) ? 0.f : ex2(sc[i] - m_mine);
          psum += pv[i];
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 16);
#pragma unroll
        for (int h = 0; h < G; ++h) l[h] += __shfl_sync(0xffffffffu, psum, h << SHIFT);
        if ((sub & ((1 << SHIFT) - 1)) == 0) {
#pragma unroll
          for (int i = 0; i < NI; ++i) pbuf[warp][i][half][my_head] = pv[i];
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < NI; ++i) {
          float vf[8];
          bf16x8_to_f32(vr[i], vf);
          float pp[G];
#pragma unroll
          for (int h = 0; h < G; ++h) pp[h] = pbuf[warp][i][half][h];
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(pp[h], vf[e], acc[h][e]);
        }
        __syncwarp();
      }
    }
    // the two half-warps accumulated different tokens of the same slices
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], 16);
    if (half == 0) {
      const size_t base = (static_cast<size_t>(b) * p.nsplit + split) * p.Hq + hq0;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (base + h) * kDecD + sub * 8);
        dst[0] = make_float4(acc[h][0] * inv, acc[h][1] * inv, acc[h][2] * inv, acc[h][3] * inv);
        dst[1] = make_float4(acc[h][4] * inv, acc[h][5] * inv, acc[h][6] * inv, acc[h][7] * inv);
        if (sub == 0)
          p.ws_lse[base + h] = l[h] > 0.f ? (m[h] + __log2f(l[h])) * kLn2 : -INFINITY;
      }
    }
  }
}

// One CTA of 128 threads per (sequence, query head); thread d owns output column d.
__global__ void __launch_bounds__(kDecD) fa_decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int d = threadIdx.x;
  const int len = checked_len(p, b);
  const int npages = len > 0 ? (len + kPage - 1) / kPage : 0;
  const int ns = (npages + p.pps - 1) / p.pps;
  float out = 0.f, lse = -INFINITY;
  if (ns > 0) {
    const size_t base = static_cast<size_t>(b) * p.nsplit * p.Hq + h;
    float mx = -INFINITY;
    for (int s = 0; s < ns; ++s) mx = fmaxf(mx, p.ws_lse[base + static_cast<size_t>(s) * p.Hq]);
    if (mx > -INFINITY) {
      float wsum = 0.f, acc = 0.f;
      for (int s = 0; s < ns; ++s) {
        const size_t idx = base + static_cast<size_t>(s) * p.Hq;
        const float ls = p.ws_lse[idx];
        const float w = (ls == -INFINITY) ? 0.f : ex2((ls - mx) * kLog2e);
        wsum += w;
        acc = fmaf(w, p.ws_o[idx * kDecD + d], acc);
      }
      out = acc / wsum;
      lse = mx + __log2f(wsum) * kLn2;
    }
  }
  uint32_t packed = pack_bf16x2(out, 0.f);
  p.o[static_cast<size_t>(bh) * kDecD + d] = static_cast<uint16_t>(packed & 0xffffu);
  if (p.lse && d == 0) p.lse[bh] = lse;
}

struct DevicePool {
  cudaMemPool_t pool = nullptr;
};
std::mutex g_pool_mu;
std::vector<DevicePool> g_pools;

int get_pool(int device, cudaMemPool_t* out) {
  std::lock_guard<std::mutex> g(g_pool_mu);
  if (static_cast<int>(g_pools.size()) <= device) g_pools.resize(device + 1);
  if (!g_pools[device].pool) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = device;
    cudaMemPool_t pool;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess)
      return set_error(FA_ERR_CUDA, "cudaMemPoolCreate: %s", cudaGetErrorString(e));
    uint64_t keep = ~0ull;   // keep freed workspace cached in the pool between calls
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pools[device].pool = pool;
  }
  *out = g_pools[device].pool;
  return FA_OK;
}

template <int G>
int launch_split(const DecodeParams& prm, cudaStream_t stream) {
  dim3 grid(prm.nsplit, prm.B);
  fa_decode_split_kernel<G><<<grid, kDecThreads, 0, stream>>>(prm);
  return FA_OK;
}

}  // namespace

int launch_decode(const void* q, const void* kcache, const void* vcache, const int32_t* block_table,
                  const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                  int page_size, float scale, int max_pages_per_seq, int num_pages,
                  cudaStream_t stream, int device) {
  if (D != kDecD) return set_error(FA_ERR_UNSUPPORTED, "decode supports D == 128 only (got %d)", D);
  if (page_size != kPage)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports page_size == 16 only (got %d)", page_size);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} (got %d)", G);
  DecodeParams prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.kc = static_cast<const uint16_t*>(kcache);
  prm.vc = static_cast<const uint16_t*>(vcache);
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.o = static_cast<uint16_t*>(o);
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.max_pages = max_pages_per_seq;
  prm.num_pages = num_pages;
  // Pages per split: aim at ~2048 CTAs if every sequence were full length.
  long long want = (static_cast<long long>(B) * max_pages_per_seq + 2047) / 2048;
  int pps = 4;
  while (pps < want && pps < 64) pps *= 2;
  prm.pps = pps;
  prm.nsplit = (max_pages_per_seq + pps - 1) / pps;
  prm.scale_log2 = scale * kLog2e;
  prm.err = device_error_word(device);
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  if (prm.nsplit > 65535 || B > 65535)
    return set_error(FA_ERR_UNSUPPORTED, "too many sequences or splits for one launch");

  const size_t n_part = static_cast<size_t>(B) * prm.nsplit * Hq;
  const size_t bytes = n_part * kDecD * sizeof(float) + n_part * sizeof(float);
  cudaMemPool_t pool;
  int rc = get_pool(device, &pool);
  if (rc != FA_OK) return rc;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, bytes, pool, stream);
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "workspace allocation (%zu bytes): %s", bytes,
                     cudaGetErrorString(e));
  prm.ws_o = static_cast<float*>(ws);
  prm.ws_lse = prm.ws_o + n_part * kDecD;
  switch (G) {
    case 1: launch_split<1>(prm, stream); break;
    case 2: launch_split<2>(prm, stream); break;
    case 4: launch_split<4>(prm, stream); break;
    default: launch_split<8>(prm, stream); break;
  }
  fa_decode_combine_kernel<<<B * Hq, kDecD, 0, stream>>>(prm);
  e = cudaGetLastError();
  cudaError_t ef = cudaFreeAsync(ws, stream);
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  if (ef != cudaSuccess)
    return set_error(FA_ERR_CUDA, "workspace release: %s", cudaGetErrorString(ef));
  return FA_OK;
}

void release_decode_resources() {
  std::lock_guard<std::mutex> g(g_pool_mu);
  for (auto& dp : g_pools) {
    if (dp.pool) {
      cudaMemPoolDestroy(dp.pool);
      dp.pool = nullptr;
    }
  }
}

}  // namespace fa

// ---------------------------------------------------------------- no-allocation variant
//
// Same split and combine kernels as launch_decode, but the chunk partials live
// in a fixed array compiled into this library instead of memory obtained at
// call time, for callers that cannot allocate device memory during a decode
// step.  The array is part of the library's device image: every GPU on which
// the library's kernels are loaded holds these bytes until the process exits.
// Every call shares it and it keeps the previous call's contents; nothing in it
// has to start at zero, because the merge only reads chunk results written
// earlier in the same call.  Two calls whose kernels overlap on the GPU (for
// example on two streams) use the same bytes and race.
namespace fa {

static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
std::mutex g_scratch_mu;
float* g_scratch_ptr[64] = {};

// Device address of g_decode_scratch on `device` (which must be current).  In
// host code the array's name is only a host-side stand-in; the address a kernel
// may use comes from cudaGetSymbolAddress, looked up once per device.
int scratch_address(int device, float** out) {
  if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(FA_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s",
                       cudaGetErrorString(e));
    g_scratch_ptr[device] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[device];
  return FA_OK;
}
}  // namespace

int plan_decode_noalloc(int B, int Hq, int max_pages_per_seq, int* pps_out, int* nsplit_out) {
  // Start from the split size launch_decode would use and widen the splits
  // until the partials fit the fixed scratch array.
  long long want = (static_cast<long long>(B) * max_pages_per_seq + 2047) / 2048;
  long long pps = 4;
  while (pps < want && pps < 64) pps *= 2;
  for (;;) {
    const long long nsplit = (max_pages_per_seq + pps - 1) / pps;
    const long long bytes = static_cast<long long>(B) * nsplit * Hq * (kDecD + 1) * 4;
    if (bytes <= static_cast<long long>(kNoAllocScratchBytes)) {
      *pps_out = static_cast<int>(pps);
      *nsplit_out = static_cast<int>(nsplit);
      return FA_OK;
    }
    if (nsplit == 1)
      return set_error(FA_ERR_INVALID_ARG,
                       "fa_decode_paged_noalloc: B * Hq = %lld needs %lld bytes of scratch even "
                       "with one chunk per sequence; the fixed scratch holds %zu bytes "
                       "(B * Hq <= %zu)",
                       static_cast<long long>(B) * Hq, bytes, kNoAllocScratchBytes,
                       kNoAllocScratchBytes / ((kDecD + 1) * 4));
    pps *= 2;
  }
}

int launch_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                          const int32_t* block_table, const int32_t* seq_lens, void* o, float* lse,
                          int B, int Hq, int Hkv, int max_pages_per_seq, int num_pages,
                          float scale, cudaStream_t stream, int device) {
  int pps = 0, nsplit = 0;
  int rc = plan_decode_noalloc(B, Hq, max_pages_per_seq, &pps, &nsplit);
  if (rc != FA_OK) return rc;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} (got %d)", G);
  float* scratch = nullptr;
  if ((rc = scratch_address(device, &scratch)) != FA_OK) return rc;
  DecodeParams prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.kc = static_cast<const uint16_t*>(kcache);
  prm.vc = static_cast<const uint16_t*>(vcache);
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.o = static_cast<uint16_t*>(o);
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.max_pages = max_pages_per_seq;
  prm.num_pages = num_pages;
  prm.pps = pps;
  prm.nsplit = nsplit;
  prm.scale_log2 = scale * kLog2e;
  prm.err = device_error_word(device);
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  if (nsplit > 65535 || B > 65535)
    return set_error(FA_ERR_UNSUPPORTED, "too many sequences or splits for one launch");
  const size_t n_part = static_cast<size_t>(B) * nsplit * Hq;
  prm.ws_o = scratch;
  prm.ws_lse = scratch + n_part * kDecD;
  switch (G) {
    case 1: launch_split<1>(prm, stream); break;
    case 2: launch_split<2>(prm, stream); break;
    case 4: launch_split<4>(prm, stream); break;
    default: launch_split<8>(prm, stream); break;
  }
  fa_decode_combine_kernel<<<B * Hq, kDecD, 0, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "decode (no-allocation) launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace fa
