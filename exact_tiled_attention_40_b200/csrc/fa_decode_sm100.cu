// Split-KV decode over a paged KV cache for sm_100a.
//
// Decode (cabseo.com, "Advanced techniques for enhancing LLM throughput",
// sections "Memory requirements" and "Autoregressive and memory-bound
// operations") attends one new query token per sequence over the whole KV
// cache, a matrix-vector product bound by HBM bandwidth.  The cache is paged
// (section "Paged attention"): fixed pages of 16 token slots, each slot holding
// all KV heads, reached through a per-sequence block table.
//
// Within a warp each half-warp takes one token and each of its 16 lanes a
// 16-byte slice (8 elements) of the 256-byte head row.  Partial dot products for
// the G query heads that share the KV head are folded across the 16 lanes with a
// transposing butterfly (each exchange halves the number of live heads), leaving
// every lane with the full score of one head.  An online softmax (running max,
// rescale by exp2(m_old - m_new), unnormalised accumulator) runs over the keys,
// and each chunk's normalised output and LSE go to a workspace that a combine
// kernel merges by LSE -- the softmax merge of unite.ai, "Flash Attention:
// Revolutionizing Transformer Efficiency", section "The Mathematics of Flash
// Attention", formula 2.
//
// Two schedules:
//  * Hkv <= 8 (streamed): one persistent CTA per SM.  All sequences' caches form
//    one list of half-pages (8 token slots: 8 * Hkv * 256 bytes of K and as many
//    of V, each contiguous in the pool); CTA c takes the equal share
//    [c*H/C, (c+1)*H/C) of the H half-pages, whatever the sequence lengths.  A
//    producer warp streams them through a shared-memory ring with TMA tensor
//    copies (128-byte swizzle, head-major boxes); eight consumer warps (warp g <-> KV head g) compute scores and
//    outputs with warp-level tensor-core MMAs from shared memory and emit one
//    partial result per (CTA, sequence) segment, stored in
//    slot c + b (unique: along the list either c or b or both grow by one); a
//    merge kernel combines each sequence's segments.
//  * otherwise (direct): grid (chunk, sequence) of fixed page chunks, cache read
//    straight from HBM with 16-byte non-allocating loads.
#include <cstdio>
#include <cstring>
#include <algorithm>
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

// streamed schedule
constexpr int kHalf = 8;                        // token slots per stage
constexpr int kConsumerWarps = kDecWarps;       // one per KV head (see the stream kernel)
constexpr int kStreamThreads = 12 * 32;          // 8 consumer warps + a producer warpgroup
// Register split (setmaxnreg): the producer warpgroup (warps 8-11, one of them
// working) gives registers to the two consumer warpgroups; 40 x 128 + 224 x 256
// stays within the 384 x 168 the block is launched with.
constexpr uint32_t kRegsProducer = 48;
constexpr uint32_t kRegsConsumer = 224;
static_assert(kRegsProducer * 128 + kRegsConsumer * 256 <= 384 * 168, "register split");
constexpr int kMaxStages = 8;
constexpr int kStreamSmemBudget = 200 * 1024;
// Streamed schedule: the half-page list is split into equal contiguous shares,
// one per CTA.  The first 15/16 of each share is streamed by its own CTA; the
// last 16th is cut into units of kDynUnit half-pages that go to whichever CTA
// asks first, so CTAs that stream more slowly (SMs differ in the bandwidth they
// get) finish with the others.  Keeping each share's units next to it spreads
// them over all sequences, so no sequence collects many partials.
constexpr int kDynDiv = 16;    // 1 / kDynDiv of each share is dynamic
constexpr int kDynUnit = 8;    // half-pages per dynamic unit (at least)
constexpr int kMaxUnitsPerCta = 4;
constexpr int kMaxStreamCtas = 204;                       // so a sequence has <= 1024 partials
constexpr int kMaxMergeSlots = kMaxStreamCtas * (1 + kMaxUnitsPerCta);
constexpr int kMergeWarps = 32;
constexpr int kHbSmemMax = 4096;   // sequences whose offsets the producer keeps in shared memory

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int32_t* block_table;
  const int32_t* seq_lens;
  uint16_t* o;
  float* lse;
  float* ws_o;     // partial outputs, [slot][Hq][128] normalised
  float* ws_lse;   // partial LSE (natural log), [slot][Hq]
  int* hb;         // streamed: hb[b] = half-pages before sequence b, hb[B] = total
  int* dyn_next;   // streamed: next dynamic unit to hand out (zeroed by the scan kernel)
  int B, Hq, Hkv, max_pages, num_pages;
  int pps, nsplit;             // direct schedule
  int nctas, nstages;          // streamed schedule
  int dyn_units_cap;           // streamed: partial slots reserved for dynamic units
  int hb_in_smem;              // streamed: the producer copies hb to shared memory
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


// A stage holds, for K and for V, two TMA boxes (head dimension halves) of
// [Hkv heads][8 tokens][64 elements] with 128-byte swizzle: the 128-byte row of
// (head g, token t) keeps its 16-byte chunk c at position c ^ t, so the 8 token
// rows of one head are read by ldmatrix without bank conflicts.
__host__ __device__ constexpr int box_bytes(int Hkv) { return Hkv * kHalf * 64 * 2; }
__host__ __device__ constexpr int stage_kv_bytes(int Hkv) { return 2 * box_bytes(Hkv); }

// hb[b] = sum over b' < b of ceil(len_b' / 8); hb[B] = total.  One block.
__global__ void __launch_bounds__(1024) fa_decode_scan_kernel(const DecodeParams p) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  pdl_launch_dependents();   // the stream kernel may launch now; it waits for hb itself
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    *p.dyn_next = 0;
  }
  __syncthreads();
  for (int base = 0; base < p.B; base += 1024) {
    const int b = base + threadIdx.x;
    int v = 0;
    if (b < p.B) {
      const int len = checked_len(p, b);
      if (len < 0)
        atomicOr(p.err, kErrBadIndex);
      else
        v = (len + kHalf - 1) / kHalf;
    }
    int x = v;   // inclusive warp scan
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += y;
      }
      warp_sums[lane] = w;   // inclusive prefix of warp totals
    }
    __syncthreads();
    const int before = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
    if (b < p.B) p.hb[b] = before;
    __syncthreads();
    if (threadIdx.x == 1023) carry = before + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.hb[p.B] = carry;
}

// CTA whose share [c*H/C, (c+1)*H/C) holds half-page x < H: the largest c with
// c*H/C <= x.
__device__ __forceinline__ int cta_of(long long x, long long H, long long C) {
  if ((x + 1) * C <= 0x7fffffffLL)             // the usual case: 32-bit division
    return static_cast<int>((static_cast<uint32_t>(x + 1) * static_cast<uint32_t>(C) - 1u) /
                            static_cast<uint32_t>(H));
  return static_cast<int>(((x + 1) * C - 1) / H);
}
// floor(c * H / C) for 0 <= c <= C
__device__ __forceinline__ int share_edge(int c, int H, int C) {
  const long long prod = static_cast<long long>(c) * H;
  if (prod <= 0x7fffffffLL)
    return static_cast<int>(static_cast<uint32_t>(prod) / static_cast<uint32_t>(C));
  return static_cast<int>(prod / C);
}

// Share of CTA c: [x0, x1) = [c*H/C, (c+1)*H/C); its own part [x0, y) and its
// dynamic part [y, x1) of d = (x1 - x0) / kDynDiv half-pages, cut into units of
// U half-pages; unit k of CTA c is global unit c * NUc + k (it may be empty).
// At most cap units in all (cap < C: no dynamic parts).  The partial of a
// segment of sequence b goes to slot c + b (own part of CTA c) or
// C + B + u + b (unit u): along the list the sequence index and the share or
// unit index never both stay the same, so the slots are distinct.
struct StreamSplit {
  int U, NUc;
};
__device__ __forceinline__ StreamSplit stream_split(int H, int C, int cap) {
  StreamSplit sp;
  sp.U = kDynUnit;
  sp.NUc = 0;
  const int per_cta = min(cap / C, kMaxUnitsPerCta);
  const int dmax = ((H + C - 1) / C) / kDynDiv;
  if (per_cta > 0 && dmax > 0) {
    if ((dmax + sp.U - 1) / sp.U > per_cta) sp.U = (dmax + per_cta - 1) / per_cta;
    sp.NUc = (dmax + sp.U - 1) / sp.U;
  }
  return sp;
}
struct Share {
  int x0, y, x1;
};
__device__ __forceinline__ Share share_of(int c, int H, int C, const StreamSplit& sp) {
  Share sh;
  sh.x0 = share_edge(c, H, C);
  sh.x1 = share_edge(c + 1, H, C);
  sh.y = sh.x1 - (sp.NUc > 0 ? (sh.x1 - sh.x0) / kDynDiv : 0);
  return sh;
}

struct StageMeta {
  int b, hh, flags, len;   // flags: 1 = first of segment, 2 = last of segment, 4 = page valid,
                           //        8 = no more stages
  int slot0;               // partial slot of this segment = slot0 + b
};

template <int G>
__global__ void __launch_bounds__(kStreamThreads, 1)
    fa_decode_stream_kernel(const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  // Consumer warp g owns KV head g and its G <= 8 query heads.  Scores and
  // outputs use warp-level tensor-core MMAs: S (16 x 8) = Q (16 query-head rows,
  // G used) x K^T per 8-token stage, then O (16 x 128) += P (16 x 8) x V; the
  // score fragment becomes the P operand in registers, and every lane's rows
  // are its own query head, so the online softmax needs no broadcasts.
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
  __shared__ StageMeta meta[kMaxStages];
  __shared__ int abort_sm;

  const int c = blockIdx.x;
  const int C = gridDim.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NS = p.nstages;
  const int HB = box_bytes(p.Hkv);              // one TMA box (half of the head dimension)
  const int SKV = stage_kv_bytes(p.Hkv);        // bytes per stage for K (and for V)
  // swizzled TMA destinations must be 1024-byte aligned
  const uint32_t sbase = (smem_u32(dsm_raw) + 1023u) & ~1023u;
  auto full = [&](int st) { return smem_u32(&bars[st]); };
  auto empty = [&](int st) { return smem_u32(&bars[kMaxStages + st]); };
  volatile int* abort_flag = &abort_sm;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), kConsumerWarps);
    }
    abort_sm = 0;
    fence_barrier_init();
  }
  // Everything above overlaps the scan kernel; the half-page offsets are its output.
  pdl_wait();
  // The merge kernel may launch once every CTA is past this point, so its launch
  // implies that the scan has finished: it reads the offsets before its own wait.
  pdl_launch_dependents();
  const int H = p.hb[p.B];
  const StreamSplit sp = stream_split(H, C, p.dyn_units_cap);
  const Share own = share_of(c, H, C, sp);
  __syncthreads();

  if (warp >= kConsumerWarps) {
    regs_dec<kRegsProducer>();
    if (warp != kConsumerWarps) return;
    // ---------------------------------------------------------------- producer
    // The sequence offsets are searched for every stage: keep them in shared
    // memory (after the stage ring) when they fit.
    const int* hbp = p.hb;
    if (p.hb_in_smem) {
      int* hb_sm = reinterpret_cast<int*>(dsm_raw + (sbase - smem_u32(dsm_raw)) + NS * 2 * SKV);
      for (int i = lane; i <= p.B; i += 32) hb_sm[i] = p.hb[i];
      __syncwarp();
      hbp = hb_sm;
    }
    // Ranges of the half-page list: this CTA's static share, then dynamic units
    // while any are left.  For each range the whole warp resolves the next 32
    // stages (sequence, half-page, page id, length) with independent loads and
    // lane 0 issues them in order.  A last stage flagged 8 ends the consumers.
    int issued = 0;
    bool ok = true;
    auto acquire_stage = [&](int& st) {
      st = issued % NS;
      return mbar_wait_sleepy(empty(st), ((issued / NS) & 1) ^ 1, abort_flag, p.err, kWaitLimitNs);
    };
    auto run_range = [&](int xs, int cnt, int slot0) {
      for (int base = 0; base < cnt && ok; base += 32) {
        const int i = base + lane;
        int bq = 0, hh = 0, page = -1, len = 0, flags = 0;
        if (i < cnt) {
          const int x = xs + i;
          int lo = 0, hi = p.B;                  // hb[lo] <= x < hb[hi]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (hbp[mid] <= x) lo = mid; else hi = mid;
          }
          bq = lo;
          const int hb_b = hbp[bq], hb_n = hbp[bq + 1];
          hh = x - hb_b;
          page = p.block_table[static_cast<size_t>(bq) * p.max_pages + (hh >> 1)];
          len = p.seq_lens[bq];
          const bool valid = page >= 0 && page < p.num_pages;
          flags = ((i == 0 || hh == 0) ? 1 : 0) | ((i == cnt - 1 || x + 1 == hb_n) ? 2 : 0) |
                  (valid ? 4 : 0);
        }
        const int cnt_here = min(32, cnt - base);
        for (int k = 0; k < cnt_here; ++k) {
          const int kb = __shfl_sync(0xffffffffu, bq, k);
          const int khh = __shfl_sync(0xffffffffu, hh, k);
          const int kpage = __shfl_sync(0xffffffffu, page, k);
          const int klen = __shfl_sync(0xffffffffu, len, k);
          const int kflags = __shfl_sync(0xffffffffu, flags, k);
          if (lane == 0) {
            int st;
            if (!acquire_stage(st)) {
              ok = false;
            } else {
              StageMeta md;
              md.b = kb;
              md.hh = khh;
              md.len = klen;
              md.flags = kflags;
              md.slot0 = slot0;
              meta[st] = md;
              if (kflags & 4) {
                const int tok0 = kpage * kPage + (khh & 1) * kHalf;
                const uint32_t kdst = sbase + st * 2 * SKV;
                mbar_arrive_expect_tx(full(st), 2 * SKV);
                tma_load_3d(kdst, &tmK, full(st), 0, tok0, 0);
                tma_load_3d(kdst + HB, &tmK, full(st), 64, tok0, 0);
                tma_load_3d(kdst + SKV, &tmV, full(st), 0, tok0, 0);
                tma_load_3d(kdst + SKV + HB, &tmV, full(st), 64, tok0, 0);
              } else {
                atomicOr(p.err, kErrBadIndex);   // consumers skip this stage
                mbar_arrive(full(st));
              }
              ++issued;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
      }
    };
    if (own.y > own.x0) run_range(own.x0, own.y - own.x0, c);
    const int n_units = C * sp.NUc;
    while (ok && n_units > 0) {
      int u = 0;
      if (lane == 0) u = atomicAdd(p.dyn_next, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= n_units) break;
      const Share sh = share_of(u / sp.NUc, H, C, sp);
      const int xs = sh.y + (u % sp.NUc) * sp.U;
      if (xs < sh.x1) run_range(xs, min(sh.x1, xs + sp.U) - xs, C + p.B + u);
    }
    if (lane == 0) {
      int st;
      if (ok && acquire_stage(st)) {             // end marker: no copy behind it
        StageMeta md;
        md.b = 0;
        md.hh = 0;
        md.len = 0;
        md.flags = 8;
        md.slot0 = 0;
        meta[st] = md;
        mbar_arrive(full(st));
        ++issued;
      }
      // copies still in flight must land before the CTA exits
      volatile int no_abort = 0;
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait(full(i % NS), (i / NS) & 1, &no_abort, p.err, kWaitLimitNs);
    }
    return;
  }

  regs_inc<kRegsConsumer>();
  // ------------------------------------------------------------------ consumers
  // Fragment layout (m16n8k16 / m16n8k8, gq = lane / 4, tq = lane % 4): score and
  // output rows are query heads gq (rows gq + 8 are unused and stay zero),
  // columns are tokens 2 tq, 2 tq + 1 of the stage (scores) or output columns
  // 8 n + 2 tq, 8 n + 2 tq + 1 (chunk n of O).
  const int gq = lane >> 2;
  const int tq = lane & 3;
  const int g = warp;                          // KV head of this warp (idle when g >= Hkv)
  const bool active = g < p.Hkv;
  const bool my_row = gq < G;                  // this lane's rows are real query heads
  const int hq = g * G + (my_row ? gq : 0);
  uint32_t qa[8][2];                           // Q A-fragments per 16-wide d chunk
  float o[16][4];
  float m_run = -INFINITY, l_run = 0.f;
  // ldmatrix: lane supplies row (head g, token lane % 8) of matrix lane / 8; for the
  // 32-wide group dg that is swizzled chunk ((dg & 1) * 4 + lane / 8) ^ (lane % 8)
  // in box dg / 2.
  const int lt = lane & 7;
  const uint32_t row_off = static_cast<uint32_t>((g * kHalf + lt) * 128);
  uint32_t ld_off[4];
#pragma unroll
  for (int dg = 0; dg < 4; ++dg)
    ld_off[dg] = static_cast<uint32_t>((dg >> 1) * HB) + row_off +
                 static_cast<uint32_t>((((dg & 1) * 4 + (lane >> 3)) ^ lt) << 4);
  for (int i = 0;; ++i) {
    const int st = i % NS;
    const bool ready = mbar_wait(full(st), (i / NS) & 1, abort_flag, p.err, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ready)) return;
    const StageMeta md = meta[st];
    if (md.flags & 8) break;                   // the producer has no more stages
    if (active) {
      if (md.flags & 1) {                      // a new sequence segment begins
        m_run = -INFINITY;
        l_run = 0.f;
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
            p.q + (static_cast<size_t>(md.b) * p.Hq + hq) * kDecD);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          qa[kc][0] = my_row ? qrow[kc * 8 + tq] : 0u;       // elements 16 kc + 2 tq, +1
          qa[kc][1] = my_row ? qrow[kc * 8 + 4 + tq] : 0u;   // elements 16 kc + 8 + 2 tq, +1
        }
#pragma unroll
        for (int nn = 0; nn < 16; ++nn) o[nn][0] = o[nn][1] = o[nn][2] = o[nn][3] = 0.f;
      }
      if (md.flags & 4) {
        const int ntok = min(kHalf, md.len - md.hh * kHalf);
        const uint32_t kaddr = sbase + st * 2 * SKV;
        const uint32_t vaddr = kaddr + SKV;
        // S = Q K^T over the 128-wide head dimension, 32 columns per ldmatrix
        float sa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int dg = 0; dg < 4; ++dg) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kaddr + ld_off[dg], b0, b1, b2, b3);
          mma_bf16_16816(sa, qa[2 * dg][0], 0u, qa[2 * dg][1], 0u, b0, b1);
          mma_bf16_16816(sa, qa[2 * dg + 1][0], 0u, qa[2 * dg + 1][1], 0u, b2, b3);
        }
        const int t0 = 2 * tq;
        const float s0 = t0 < ntok ? sa[0] * p.scale_log2 : -INFINITY;
        const float s1 = t0 + 1 < ntok ? sa[1] * p.scale_log2 : -INFINITY;
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
        m_run = m_new;
        const float p0 = (s0 == -INFINITY) ? 0.f : ex2(s0 - m_run);
        const float p1 = (s1 == -INFINITY) ? 0.f : ex2(s1 - m_run);
        l_run = l_run * alpha + (p0 + p1);
        const uint32_t pa = pack_bf16x2(p0, p1);   // P A-fragment: row gq, tokens 2 tq, 2 tq + 1
#pragma unroll
        for (int nn = 0; nn < 16; ++nn) {
          o[nn][0] *= alpha;
          o[nn][1] *= alpha;
        }
#pragma unroll
        for (int ng = 0; ng < 4; ++ng) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_t(vaddr + ld_off[ng], v0, v1, v2, v3);
          mma_bf16_1688(o[4 * ng + 0], pa, 0u, v0);
          mma_bf16_1688(o[4 * ng + 1], pa, 0u, v1);
          mma_bf16_1688(o[4 * ng + 2], pa, 0u, v2);
          mma_bf16_1688(o[4 * ng + 3], pa, 0u, v3);
        }
      }

      if (md.flags & 2) {                      // segment ends: its partial goes to slot0 + b
        float l_tot = l_run;
        l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 1);
        l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
        if (my_row) {
          const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
          const size_t rowi = (static_cast<size_t>(md.slot0) + md.b) * p.Hq + hq;
          float* dst = p.ws_o + rowi * kDecD + 2 * tq;
#pragma unroll
          for (int nn = 0; nn < 16; ++nn)
            *reinterpret_cast<float2*>(dst + 8 * nn) = make_float2(o[nn][0] * inv, o[nn][1] * inv);
          if (tq == 0)
            p.ws_lse[rowi] = l_tot > 0.f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }
}

// Streamed schedule, merge: one block per sequence b.  The partials of b sit in
// slot c + b for every CTA c whose own part meets b, and in slot C + B + u + b
// for every dynamic unit u that meets b; warp 0 lists them in shared memory
// (lanes over CTAs), then each warp merges query heads by their LSE (formula 2
// of the softmax merge), lane i owning output columns [4i, 4i + 4).
//
// The offsets are the scan kernel's output, which has finished by the time this
// grid launches (the stream kernel signals its dependents only after its own
// wait on the scan), so the slot list is built while the stream kernel still
// runs; after the wait only the partials are read, the LSEs and the first
// kMergeBatch partial rows of a head in one round of independent loads.
constexpr int kMergeBatch = 8;

__global__ void __launch_bounds__(kMergeWarps * 32) fa_decode_stream_merge_kernel(
    const DecodeParams p) {
  __shared__ int slots[kMaxMergeSlots];
  __shared__ int n_slots_sm;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int xs = __ldcg(p.hb + b), xe = __ldcg(p.hb + b + 1);
  if (xe <= xs) {                              // no keys (or an invalid length): O = 0, LSE = -inf
    pdl_wait();
    for (int h = warp; h < p.Hq; h += kMergeWarps) {
      const size_t wid = static_cast<size_t>(b) * p.Hq + h;
      *reinterpret_cast<uint2*>(p.o + wid * kDecD + lane * 4) = make_uint2(0, 0);
      if (p.lse && lane == 0) p.lse[wid] = -INFINITY;
    }
    return;
  }
  const int H = __ldcg(p.hb + p.B);
  const int C = p.nctas;
  const StreamSplit sp = stream_split(H, C, p.dyn_units_cap);
  if (warp == 0) {
    const int c_first = cta_of(xs, H, C), c_last = cta_of(xe - 1, H, C);
    int base = 0;
    for (int c0 = c_first; c0 <= c_last; c0 += 32) {
      const int cc = c0 + lane;
      Share sh;
      int own = 0, k0 = 0, k1 = -1;
      if (cc <= c_last) {
        sh = share_of(cc, H, C, sp);
        own = max(xs, sh.x0) < min(xe, sh.y) ? 1 : 0;
        const int lo = max(xs, sh.y), hi = min(xe, sh.x1);
        if (lo < hi) {
          k0 = (lo - sh.y) / sp.U;
          k1 = (hi - 1 - sh.y) / sp.U;
        }
      }
      const int cnt = own + (k1 - k0 + 1);
      int incl = cnt;                          // inclusive prefix over the lanes
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
      }
      int at = base + incl - cnt;
      if (own && at < kMaxMergeSlots) slots[at] = cc + b;
      at += own;
      for (int k = k0; k <= k1; ++k, ++at)
        if (at < kMaxMergeSlots) slots[at] = C + p.B + cc * sp.NUc + k + b;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) n_slots_sm = min(base, kMaxMergeSlots);
  }
  __syncthreads();
  const int ns = n_slots_sm;
  pdl_wait();                                  // the stream kernel's partials
  const float4* wo = reinterpret_cast<const float4*>(p.ws_o);
  auto row = [&](int k, int h) {               // lane's four columns of slot k, head h
    return __ldcg(wo + (static_cast<size_t>(slots[k]) * p.Hq + h) * (kDecD / 4) + lane);
  };
  for (int h = warp; h < p.Hq; h += kMergeWarps) {
    // 32 slots at a time (one sequence rarely has more): one LSE per lane and the
    // first kMergeBatch rows load together; a later chunk with a larger maximum
    // rescales what is accumulated so far
    float wsum = 0.f, mx = -INFINITY;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < ns; k0 += 32) {
      const int cnt = min(32, ns - k0);
      const float ls =
          lane < cnt ? __ldcg(p.ws_lse + static_cast<size_t>(slots[k0 + lane]) * p.Hq + h)
                     : -INFINITY;
      float4 v[kMergeBatch];
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j)
        if (j < cnt) v[j] = row(k0 + j, h);
      float m = ls;
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
      m = fmaxf(m, mx);
      if (m == -INFINITY) continue;            // every LSE so far is -inf (warp-uniform)
      const float sc = ex2((mx - m) * kLog2e); // 0 on the first finite chunk
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
      wsum *= sc;
      mx = m;
      const float w = (ls == -INFINITY) ? 0.f : ex2((ls - mx) * kLog2e);
      wsum += w;
      for (int j0 = 0; j0 < cnt; j0 += kMergeBatch) {
        if (j0 > 0) {
#pragma unroll
          for (int j = 0; j < kMergeBatch; ++j)
            if (j0 + j < cnt) v[j] = row(k0 + j0 + j, h);
        }
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
          const float wj = __shfl_sync(0xffffffffu, w, (j0 + j) & 31);
          if (j0 + j < cnt) {
            acc.x = fmaf(wj, v[j].x, acc.x);
            acc.y = fmaf(wj, v[j].y, acc.y);
            acc.z = fmaf(wj, v[j].z, acc.z);
            acc.w = fmaf(wj, v[j].w, acc.w);
          }
        }
      }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, d);
    const size_t wid = static_cast<size_t>(b) * p.Hq + h;
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    *reinterpret_cast<uint2*>(p.o + wid * kDecD + lane * 4) =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    if (p.lse && lane == 0) p.lse[wid] = wsum > 0.f ? mx + __log2f(wsum) * kLn2 : -INFINITY;
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

int sm_count(int device) {
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

// Launch geometry and workspace size of one decode call.
struct DecodePlan {
  bool streamed = false;
  int pps = 0, nsplit = 0;     // direct schedule
  int nctas = 0, nstages = 0;  // streamed schedule
  int dyn_units_cap = 0;       // streamed: dynamic units the partial slots allow
  size_t n_part = 0;           // partial rows (slot x head)
  size_t bytes = 0;            // workspace bytes
};

// Direct schedule: pages per chunk so that a full-length batch makes ~2048 CTAs.
int direct_pps(int B, int max_pages_per_seq) {
  const long long want = (static_cast<long long>(B) * max_pages_per_seq + 2047) / 2048;
  int pps = 4;
  while (pps < want && pps < 64) pps *= 2;
  return pps;
}

void finish_plan(DecodePlan& pl, int B, int Hq, int Hkv) {
  if (pl.streamed) {
    // slots: C + B static, then (units + B) dynamic when there are units
    const size_t dyn_slots = pl.dyn_units_cap > 0 ? static_cast<size_t>(pl.dyn_units_cap) + B : 0;
    pl.n_part = (static_cast<size_t>(pl.nctas) + B + dyn_slots) * Hq;
    pl.bytes = pl.n_part * (kDecD + 1) * sizeof(float) + (static_cast<size_t>(B) + 2) * sizeof(int);
  } else {
    pl.n_part = static_cast<size_t>(B) * pl.nsplit * Hq;
    pl.bytes = pl.n_part * (kDecD + 1) * sizeof(float);
  }
}

DecodePlan make_plan(int B, int Hq, int Hkv, int max_pages_per_seq, int nsm) {
  DecodePlan pl;
  // streamed: one consumer warp per KV head, its G <= 8 query heads as MMA rows
  pl.streamed = Hkv <= kDecWarps && nsm > 0;
  if (pl.streamed) {
    pl.nctas = std::min(nsm, kMaxStreamCtas);
    pl.nstages = kStreamSmemBudget / (2 * stage_kv_bytes(Hkv));
    if (pl.nstages > kMaxStages) pl.nstages = kMaxStages;
    // enough units for the dynamic part of every share of the longest possible list
    const long long h_max = 2LL * B * max_pages_per_seq;
    const long long per_cta = ((h_max + pl.nctas - 1) / pl.nctas) / kDynDiv / kDynUnit + 1;
    pl.dyn_units_cap = static_cast<int>(std::min<long long>(per_cta * pl.nctas, 1 << 24));
  } else {
    pl.pps = direct_pps(B, max_pages_per_seq);
    pl.nsplit = (max_pages_per_seq + pl.pps - 1) / pl.pps;
  }
  finish_plan(pl, B, Hq, Hkv);
  return pl;
}

template <int G>
int launch_kernels(const DecodeParams& prm, const DecodePlan& pl, const CUtensorMap& tmK,
                   const CUtensorMap& tmV, cudaStream_t stream, int device) {
  if (pl.streamed) {
    const int smem = pl.nstages * 2 * stage_kv_bytes(prm.Hkv) + 1024 +
                     (prm.hb_in_smem ? (prm.B + 1) * 4 : 0);
    {
      // the shared-memory limit is a property of the function on each device
      static int attr_gen[64] = {};
      static std::mutex mu;
      std::lock_guard<std::mutex> g(mu);
      if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
      if (attr_gen[device] != cache_generation()) {
        cudaError_t e = cudaFuncSetAttribute(fa_decode_stream_kernel<G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kStreamSmemBudget + 1024 + kHbSmemMax * 4);
        if (e != cudaSuccess)
          return set_error(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_gen[device] = cache_generation();
      }
    }
    // The stream and merge kernels are launched with programmatic serialization:
    // each may start while its predecessor runs and waits (griddepcontrol.wait)
    // before it reads the predecessor's output, which hides the launch gaps.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    fa_decode_scan_kernel<<<1, 1024, 0, stream>>>(prm);
    cfg.gridDim = dim3(pl.nctas);
    cfg.blockDim = dim3(kStreamThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchKernelEx(&cfg, fa_decode_stream_kernel<G>, tmK, tmV, prm);
    cfg.gridDim = dim3(prm.B);
    cfg.blockDim = dim3(kMergeWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cudaLaunchKernelEx(&cfg, fa_decode_stream_merge_kernel, prm);
  } else {
    dim3 grid(pl.nsplit, prm.B);
    fa_decode_split_kernel<G><<<grid, kDecThreads, 0, stream>>>(prm);
    fa_decode_combine_kernel<<<prm.B * prm.Hq, kDecD, 0, stream>>>(prm);
  }
  return FA_OK;
}

// Runs one decode with the given workspace (at least pl.bytes, 256-byte aligned).
int run_decode(const void* q, const void* kcache, const void* vcache, const int32_t* block_table,
               const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv,
               int max_pages_per_seq, int num_pages, float scale, const DecodePlan& pl, void* ws,
               cudaStream_t stream, int device) {
  const int G = Hq / Hkv;
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
  prm.pps = pl.pps;
  prm.nsplit = pl.nsplit;
  prm.nctas = pl.nctas;
  prm.nstages = pl.nstages;
  prm.dyn_units_cap = pl.dyn_units_cap;
  prm.hb_in_smem = B + 1 <= kHbSmemMax ? 1 : 0;
  prm.scale_log2 = scale * kLog2e;
  prm.err = device_error_word(device);
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  if (!pl.streamed && (pl.nsplit > 65535 || B > 65535))
    return set_error(FA_ERR_UNSUPPORTED, "too many sequences or chunks for one launch");
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return set_error(FA_ERR_UNSUPPORTED, "B * Hq too large");
  prm.ws_o = static_cast<float*>(ws);
  prm.ws_lse = prm.ws_o + pl.n_part * kDecD;
  prm.hb = reinterpret_cast<int*>(prm.ws_lse + pl.n_part);
  prm.dyn_next = prm.hb + (B + 1);
  CUtensorMap tmK, tmV;
  if (pl.streamed) {
    // K and V caches viewed as [Hkv][num_pages * 16 tokens][128]: box {64, 8, Hkv}
    const uint64_t dims[3] = {static_cast<uint64_t>(kDecD),
                              static_cast<uint64_t>(num_pages) * kPage,
                              static_cast<uint64_t>(Hkv)};
    const uint64_t strides[2] = {static_cast<uint64_t>(Hkv) * kDecD * 2,
                                 static_cast<uint64_t>(kDecD) * 2};
    const uint32_t box[3] = {64, static_cast<uint32_t>(kHalf), static_cast<uint32_t>(Hkv)};
    int rc = encode_tensor_map_16bit(&tmK, kcache, true, 3, dims, strides, box);
    if (rc == FA_OK) rc = encode_tensor_map_16bit(&tmV, vcache, true, 3, dims, strides, box);
    if (rc != FA_OK) return rc;
  } else {
    memset(&tmK, 0, sizeof(tmK));
    memset(&tmV, 0, sizeof(tmV));
  }
  int lrc;
  switch (G) {
    case 1: lrc = launch_kernels<1>(prm, pl, tmK, tmV, stream, device); break;
    case 2: lrc = launch_kernels<2>(prm, pl, tmK, tmV, stream, device); break;
    case 4: lrc = launch_kernels<4>(prm, pl, tmK, tmV, stream, device); break;
    default: lrc = launch_kernels<8>(prm, pl, tmK, tmV, stream, device); break;
  }
  if (lrc != FA_OK) return lrc;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
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
  const DecodePlan pl = make_plan(B, Hq, Hkv, max_pages_per_seq, sm_count(device));
  cudaMemPool_t pool;
  int rc = get_pool(device, &pool);
  if (rc != FA_OK) return rc;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, pl.bytes, pool, stream);
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "workspace allocation (%zu bytes): %s", pl.bytes,
                     cudaGetErrorString(e));
  rc = run_decode(q, kcache, vcache, block_table, seq_lens, o, lse, B, Hq, Hkv, max_pages_per_seq,
                  num_pages, scale, pl, ws, stream, device);
  cudaError_t ef = cudaFreeAsync(ws, stream);
  if (rc != FA_OK) return rc;
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
// Same kernels as launch_decode, but the chunk partials live in a fixed array
// compiled into this library instead of memory obtained at call time, for
// callers that cannot allocate device memory during a decode step.  The array
// is part of the library's device image: every GPU on which the library's
// kernels are loaded holds these bytes until the process exits.  Every call
// shares it and it keeps the previous call's contents; nothing in it has to
// start at zero when the call begins: each call writes everything it later reads
// (the prefix offsets and every partial the merge reads).  Two calls whose kernels
// overlap on the GPU (for example on two streams) use the same bytes and race.
namespace fa {

static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
std::mutex g_scratch_mu;
float* g_scratch_ptr[64] = {};
int g_scratch_gen[64] = {};

// Device address of g_decode_scratch on `device` (which must be current).  In
// host code the array's name is only a host-side stand-in; the address a kernel
// may use comes from cudaGetSymbolAddress, looked up once per device (and again
// after fa_release(), which a caller makes after resetting the device).
int scratch_address(int device, float** out) {
  if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> g(g_scratch_mu);
  const int gen = cache_generation();
  if (!g_scratch_ptr[device] || g_scratch_gen[device] != gen) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(FA_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s",
                       cudaGetErrorString(e));
    g_scratch_ptr[device] = static_cast<float*>(p);
    g_scratch_gen[device] = gen;
  }
  *out = g_scratch_ptr[device];
  return FA_OK;
}

// Direct schedule with its page chunks widened until the partials fit.
DecodePlan widen_direct(int B, int Hq, int Hkv, int max_pages_per_seq) {
  DecodePlan pl;
  pl.streamed = false;
  pl.pps = direct_pps(B, max_pages_per_seq);
  pl.nsplit = (max_pages_per_seq + pl.pps - 1) / pl.pps;
  finish_plan(pl, B, Hq, Hkv);
  while (pl.bytes > kNoAllocScratchBytes && pl.nsplit > 1) {
    pl.pps *= 2;
    pl.nsplit = (max_pages_per_seq + pl.pps - 1) / pl.pps;
    finish_plan(pl, B, Hq, Hkv);
  }
  return pl;
}

// Plan that fits the fixed scratch on a device with `nsm` SMs (0: no device
// known, which plans the direct schedule, the one with the smallest need).
// The streamed schedule (Hkv <= 8) is kept when it fits, if need be with fewer
// dynamic units (each then covers more half-pages) or none; otherwise the
// direct schedule with widened chunks, which needs only B * Hq rows at one
// chunk per sequence.
int plan_noalloc(int B, int Hq, int Hkv, int max_pages_per_seq, int nsm, DecodePlan* out) {
  DecodePlan pl = make_plan(B, Hq, Hkv, max_pages_per_seq, nsm);
  if (pl.streamed && pl.bytes > kNoAllocScratchBytes) {
    const long long rows_fit =
        (static_cast<long long>(kNoAllocScratchBytes) - (static_cast<long long>(B) + 2) * 4) /
        ((kDecD + 1) * 4) / Hq;
    const long long cap = rows_fit - pl.nctas - 2LL * B;
    pl.dyn_units_cap = cap > 0 ? static_cast<int>(std::min<long long>(cap, pl.dyn_units_cap)) : 0;
    finish_plan(pl, B, Hq, Hkv);
  }
  if (pl.bytes > kNoAllocScratchBytes) pl = widen_direct(B, Hq, Hkv, max_pages_per_seq);
  if (pl.bytes > kNoAllocScratchBytes)
    return set_error(FA_ERR_INVALID_ARG,
                     "fa_decode_paged_noalloc: this problem needs %zu bytes of scratch; the fixed "
                     "scratch holds %zu bytes (partial rows of %d bytes: at least B * Hq = %lld)",
                     pl.bytes, kNoAllocScratchBytes, (kDecD + 1) * 4,
                     static_cast<long long>(B) * Hq);
  *out = pl;
  return FA_OK;
}
}  // namespace

int check_decode_noalloc(int B, int Hq, int Hkv, int max_pages_per_seq, int nsm) {
  DecodePlan pl;
  return plan_noalloc(B, Hq, Hkv, max_pages_per_seq, nsm, &pl);
}

int launch_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                          const int32_t* block_table, const int32_t* seq_lens, void* o, float* lse,
                          int B, int Hq, int Hkv, int max_pages_per_seq, int num_pages,
                          float scale, cudaStream_t stream, int device) {
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(FA_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} (got %d)", G);
  DecodePlan pl;
  int rc = plan_noalloc(B, Hq, Hkv, max_pages_per_seq, sm_count(device), &pl);
  if (rc != FA_OK) return rc;
  float* scratch = nullptr;
  if ((rc = scratch_address(device, &scratch)) != FA_OK) return rc;
  return run_decode(q, kcache, vcache, block_table, seq_lens, o, lse, B, Hq, Hkv,
                    max_pages_per_seq, num_pages, scale, pl, scratch, stream, device);
}

}  // namespace fa
