// Exact attention backward for sm_100a, with recomputation.
//
// unite.ai, "Flash Attention: Revolutionizing Transformer Efficiency", names
// recomputation in the backward pass (the N x N probabilities are not stored;
// the forward keeps only O and the per-row log-sum-exp, from which P is rebuilt
// tile by tile).  With P = exp(scale Q K^T - LSE) and the row sums
// delta_i = sum_d dO_id O_id:
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),
//     dQ = scale dS K,  dK = scale dS^T Q,
// GQA: the query heads of one KV head add into its dK, dV.
//
// Three kernels, no atomics and no workspace beyond delta:
//   fa_bwd_delta_kernel  delta = rowsum(dO * O) (a warp per row, HBM-bound).
//   fa_bwd_dkdv_kernel   one CTA per (sequence, KV head, 128-key tile j): K_j, V_j
//                        stay in shared memory; the Q_i, dO_i tiles of every query
//                        head of the group stream through a two-slot ring.  Per
//                        tile pair the MMA warp computes S^T = K_j Q_i^T and
//                        dP^T = V_j dO_i^T into TMEM; the 128 softmax threads
//                        (thread r = key r = TMEM lane r) rebuild P^T and dS^T and
//                        write them back over the first halves of those TMEM
//                        columns as bf16 pairs; the MMA warp then accumulates
//                        dV += P^T dO_i and dK += dS^T Q_i (A operand from TMEM).
//   fa_bwd_dq_kernel     one CTA per (sequence, query head, 128-row tile i): Q_i,
//                        dO_i stay; K_j, V_j stream.  S = Q_i K_j^T and
//                        dP = dO_i V_j^T into TMEM, dS (per row: its own LSE and
//                        delta) back as bf16, dQ += dS K_j.
// Each recomputes S and dP, seven tile products per pair instead of five, in
// exchange for no atomics and a TMEM budget that fits (dK/dV kernel: S^T, dP^T,
// dV, dK = 4 x 128 columns at D = 128; dQ kernel: S, dP, dQ).
// Warps: 0-3 softmax (one TMEM lane quarter each), 4 TMA producer, 5 MMA issuer
// (an elected lane issues).  Every wait is bounded (mbar_wait).
#include <algorithm>
#include <cfloat>
#include <cstdio>
#include <mutex>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {
namespace {

constexpr int kBM = 128;                  // rows of every tile (TMEM lanes)
constexpr int kHalfN = 64;                // columns of a softmax warpgroup's half tile
constexpr int kThreads = 320;             // 2 x 4 softmax warps, producer, MMA
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdLayout {
  static constexpr int kChunks = D / 64;                // 128-byte swizzle atoms along D
  static constexpr int kChunkBytes = kBM * 128;
  static constexpr int kTileBytes = kBM * D * 2;
  // two stationary tiles, then a two-slot ring of tile pairs
  static constexpr int kFixOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + 4 * kTileBytes;
  static constexpr int kNumBars = 1 + 2 + 2 + 2 + 2 + 1 + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // dK/dV kernel: per warpgroup and item parity, the 64 queries' LSE (log2
  // units) and delta
  static constexpr int kStatOff = kMiscOff + 16;
  static constexpr int kStatBytes = 2 * 2 * 2 * kHalfN * 4;
  // at least 118 KB so that two CTAs never share an SM: each allocates all 512
  // TMEM columns (the next power of two above its 384 or 320 at D = 64)
  static constexpr int kSmemBytes = (kStatOff + kStatBytes + 1024) > 118 * 1024
                                        ? (kStatOff + kStatBytes + 1024)
                                        : 118 * 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct BwdParams {
  const uint16_t* o;
  const uint16_t* dout;
  const float* lse;      // [B * Hq, Nq], natural log
  float* delta;          // [B * Hq, Nq]
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  int B, Hq, Hkv, Nq, Nk;
  int causal;
  float scale;
  float scale_log2;      // scale * log2(e)
  int* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// delta[row] = sum_d dO[row, d] * O[row, d]; a warp per row.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_delta_kernel(const uint16_t* __restrict__ o,
                                                           const uint16_t* __restrict__ dout,
                                                           float* __restrict__ delta,
                                                           long long rows) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * 8;
  for (long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const size_t base = static_cast<size_t>(row) * D + lane * E;
    float acc = 0.f;
    if constexpr (E == 4) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(o + base));
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(dout + base));
      acc = bf_lo(a.x) * bf_lo(b.x) + bf_hi(a.x) * bf_hi(b.x) + bf_lo(a.y) * bf_lo(b.y) +
            bf_hi(a.y) * bf_hi(b.y);
    } else {
      const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(o + base));
      const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(dout + base));
      acc = bf_lo(a) * bf_lo(b) + bf_hi(a) * bf_hi(b);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) delta[row] = acc;
  }
}

// K-major descriptor step kk (16 elements of D) inside a [128, D] tile.
template <int D>
__device__ __forceinline__ uint64_t kmajor_step(int kk) {
  return static_cast<uint64_t>(((kk >> 2) * BwdLayout<D>::kChunkBytes + (kk & 3) * 32) >> 4);
}

// 128 x 64 product of two K-major [128, D] tiles: rows of A against rows
// row0 .. row0 + 63 of B (row0 a multiple of 64: a whole number of 8-row
// swizzle atoms), into TMEM columns d .. d + 63.
template <int D>
__device__ __forceinline__ void mma_rows_x_half(uint32_t d, uint64_t a, uint64_t b, int row0) {
  constexpr uint32_t idesc = idesc_f16(kBM, kHalfN, true, false);
  const uint64_t boff = static_cast<uint64_t>((row0 * 128) >> 4);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_ss(d, a + kmajor_step<D>(kk), b + boff + kmajor_step<D>(kk), idesc, kk > 0 ? 1u : 0u);
}

// D-column accumulation over 64 K values k0 .. k0 + 63: TMEM[d .. d + D) (+)=
// A (bf16 pairs in TMEM columns a .. a + 31) x B (rows k0 .. of a [128, D]
// tile, read MN-major).
template <int D>
__device__ __forceinline__ void mma_half_x_tile(uint32_t d, uint32_t a, uint64_t b_mn, int k0,
                                                bool accumulate) {
  constexpr uint32_t idesc = idesc_f16(kBM, D, true, true);
#pragma unroll
  for (int k = 0; k < kHalfN / 16; ++k)
    mma_ts(d, a + k * 8, b_mn + static_cast<uint64_t>(((k0 + k * 16) * 128) >> 4), idesc,
           (accumulate || k > 0) ? 1u : 0u);
}

// Store columns c0 .. c0 + ncols of a row of fp32 TMEM values (columns t0 ..),
// times `mul`, as bf16 (32 columns per step).
__device__ __forceinline__ void store_cols_bf16(uint32_t t0, int c0, int ncols, float mul,
                                                uint16_t* dst, bool valid, int* err) {
#pragma unroll 1
  for (int c = c0; c < c0 + ncols; c += 32) {
    uint32_t v[32];
    tmem_ld32(t0 + c, v, err);
    tmem_wait_ld(err);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
    if (valid) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
}

__device__ __forceinline__ void store_zero_cols(uint16_t* dst, int c0, int ncols) {
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int c = c0; c < c0 + ncols; c += 8) *reinterpret_cast<uint4*>(dst + c) = z;
}

// First query tile that sees key tile j (causal, bottom-right aligned).
__device__ __forceinline__ int first_q_tile(int j, int Nq, int Nk, int causal) {
  if (!causal) return 0;
  const int t = j * kBM - (Nk - Nq);   // the first query row that sees key j * 128
  return t <= 0 ? 0 : t / kBM;
}

// ---------------------------------------------------------------- dK, dV
// Warps 0-3 and 4-7 are two softmax warpgroups over the same 128 TMEM lanes
// (key rows): warpgroup w takes the queries 64 w .. 64 w + 63 of each tile
// pair, i.e. columns 64 w .. of S^T and 128 + 64 w .. of dP^T, and writes its
// P^T and dS^T there as 32 columns of bf16 pairs.  The MMA warp computes each
// half of S^T and dP^T with N = 64 MMAs and commits the halves separately, so
// warpgroup 0 starts while the second half is computed; dV and dK take each
// half's 64 queries as soon as its warpgroup has released it.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work: key tile j of (b, hkv); CTAs in order of j, so under the causal mask the
  // heaviest tiles (seen by the most query tiles) start first
  const int nkvh = p.B * p.Hkv;
  const int j = blockIdx.x / nkvh;
  const int bh_kv = blockIdx.x - j * nkvh;
  const int b = bh_kv / p.Hkv;
  const int hkv = bh_kv - b * p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int n_qt = (p.Nq + kBM - 1) / kBM;
  const int i0 = first_q_tile(j, p.Nq, p.Nk, p.causal);
  const int per_head = i0 < n_qt ? n_qt - i0 : 0;
  const int n_items = per_head * G;     // (query head g, query tile i0 + t)
  const int off = p.Nk - p.Nq;

  auto bar = [&](int i) -> uint32_t { return sbase + L::kBarOff + 8 * i; };
  const uint32_t kv_full = bar(0);
  auto q_full = [&](int s) { return bar(1 + s); };
  auto q_empty = [&](int s) { return bar(3 + s); };
  auto s_full = [&](int h) { return bar(5 + h); };
  auto p_full = [&](int h) { return bar(7 + h); };
  const uint32_t acc_done = bar(9);
  // a warpgroup's staged LSE and delta of one item parity are complete
  auto stat_full = [&](int w, int par) { return bar(10 + 2 * w + par); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* stat = reinterpret_cast<float*>(smem + L::kStatOff);
  const uint32_t k_smem = sbase + L::kFixOff;
  const uint32_t v_smem = sbase + L::kFixOff + L::kTileBytes;
  auto q_smem = [&](int s) { return sbase + L::kRingOff + (2 * s) * L::kTileBytes; };
  auto do_smem = [&](int s) { return sbase + L::kRingOff + (2 * s + 1) * L::kTileBytes; };

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(p_full(s), kBM);
      mbar_init(stat_full(s, 0), kBM);
      mbar_init(stat_full(s, 1), kBM);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: [0,128) S^T then P^T (warpgroup w's bf16 pairs in [64w, 64w+32));
  // [128,256) dP^T then dS^T likewise; [256,256+D) dV; [256+D,256+2D) dK

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_items > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
      const int z_kv = b * p.Hkv + hkv;
      for (int ch = 0; ch < L::kChunks; ++ch) {
        tma_load_3d(k_smem + ch * L::kChunkBytes, &tmK, kv_full, ch * 64, j * kBM, z_kv);
        tma_load_3d(v_smem + ch * L::kChunkBytes, &tmV, kv_full, ch * 64, j * kBM, z_kv);
      }
      int it = 0;
      for (; it < n_items; ++it) {
        const int s = it & 1;
        if (!mbar_wait(q_empty(s), ((it >> 1) & 1) ^ 1, abort_flag, p.err, p.timeout_ns)) break;
        const int g = it / per_head;
        const int i = i0 + (it - g * per_head);
        const int z = b * p.Hq + hkv * G + g;
        mbar_arrive_expect_tx(q_full(s), 2 * L::kTileBytes);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(q_smem(s) + ch * L::kChunkBytes, &tmQ, q_full(s), ch * 64, i * kBM, z);
          tma_load_3d(do_smem(s) + ch * L::kChunkBytes, &tmdO, q_full(s), ch * 64, i * kBM, z);
        }
      }
      // every issued copy lands before the CTA may exit
      volatile int no_abort = 0;
      mbar_wait(kv_full, 0, &no_abort, p.err, p.timeout_ns);
      for (int s = 0; s < 2 && s < it; ++s) {
        const int last = s + ((it - 1 - s) / 2) * 2;
        mbar_wait(q_full(s), (last >> 1) & 1, &no_abort, p.err, p.timeout_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    auto wait = [&](uint32_t br, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(br, parity, abort_flag, p.err, p.timeout_ns));
    };
    const uint64_t k_desc = smem_desc_sw128(k_smem, 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(v_smem, 16, 1024);
    bool ok = n_items == 0 || wait(kv_full, 0);
    for (int it = 0; ok && it < n_items; ++it) {
      const int s = it & 1;
      ok = wait(q_full(s), (it >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint64_t q_kdesc = smem_desc_sw128(q_smem(s), 16, 1024);
      const uint64_t do_kdesc = smem_desc_sw128(do_smem(s), 16, 1024);
      if (leader) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mma_rows_x_half<D>(tmem + kHalfN * h, k_desc, q_kdesc, kHalfN * h);          // S^T
          mma_rows_x_half<D>(tmem + 128 + kHalfN * h, v_desc, do_kdesc, kHalfN * h);   // dP^T
          tc_commit(s_full(h));
        }
      }
      const uint64_t q_mn = smem_desc_sw128(q_smem(s), L::kChunkBytes, 1024);
      const uint64_t do_mn = smem_desc_sw128(do_smem(s), L::kChunkBytes, 1024);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        ok = wait(p_full(h), it & 1);
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const bool acc = it > 0 || h > 0;
          mma_half_x_tile<D>(tmem + 256, tmem + kHalfN * h, do_mn, kHalfN * h, acc);        // dV
          mma_half_x_tile<D>(tmem + 256 + D, tmem + 128 + kHalfN * h, q_mn, kHalfN * h, acc);  // dK
        }
      }
      if (!ok) break;
      if (leader) tc_commit(q_empty(s));
    }
    if (leader) tc_commit(acc_done);
    volatile int no_abort = 0;
    mbar_wait(acc_done, 0, &no_abort, p.err, p.timeout_ns);
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;                           // queries 64 wg .. 64 wg + 63
    const int t = tid & 127;
    const int r = (warp & 3) * 32 + lane;               // key row within the tile
    const int kr = j * kBM + r;                         // key index
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + kHalfN * wg;
    const uint32_t tP = tmem + lane_base + 128 + kHalfN * wg;
    bool ok = true;
    for (int it = 0; ok && it < n_items; ++it) {
      const int g = it / per_head;
      const int i = i0 + (it - g * per_head);
      const size_t qrow0 = static_cast<size_t>(b * p.Hq + hkv * G + g) * p.Nq;
      const int q0 = i * kBM + kHalfN * wg;            // first query of this half
      // the half's 64 LSE (log2 units) and delta values, staged once per item in
      // a buffer of this item's parity (the buffer of item it - 2 is free: every
      // thread of the warpgroup has passed item it - 1's stat barrier)
      float* lse2_s = stat + ((wg * 2 + (it & 1)) * 2) * kHalfN;
      float* dl_s = lse2_s + kHalfN;
      {
        const int q = q0 + (t & 63);
        if (t < 64)
          lse2_s[t] = q < p.Nq ? __ldg(p.lse + qrow0 + q) * kLog2e : INFINITY;
        else
          dl_s[t - 64] = q < p.Nq ? __ldg(p.delta + qrow0 + q) : 0.f;
      }
      mbar_arrive(stat_full(wg, it & 1));
      bool got = mbar_wait(stat_full(wg, it & 1), (it >> 1) & 1, abort_flag, p.err, p.timeout_ns);
      if (got) got = mbar_wait(s_full(wg), it & 1, abort_flag, p.err, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // queries q0 + e are visible to key kr when kr <= q + off
      const bool band = p.causal && (j * kBM + kBM - 1 > q0 + off);
      const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + 32 * c, sv, p.err);
        tmem_ld32(tP + 32 * c, dv, p.err);
        tmem_wait_ld(p.err);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int ee = 32 * c + e;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2,
                           f2_pack(-lse2_s[ee], -lse2_s[ee + 1])),
                    x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (band) {
            if (kr > q0 + ee + off) p0 = 0.f;
            if (kr > q0 + ee + 1 + off) p1 = 0.f;
          }
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1),
                           f2_sub(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])),
                                  f2_pack(dl_s[ee], dl_s[ee + 1]))),
                    d0, d1);
          pk[e >> 1] = pack_bf16x2(p0, p1);
          dk[e >> 1] = pack_bf16x2(d0, d1);
        }
        // the packed pairs go over columns already read (16 c .. 16 c + 15)
        tmem_st16(tS + 16 * c, pk, p.err);
        tmem_st16(tP + 16 * c, dk, p.err);
      }
      tmem_wait_st(p.err);
      tc_fence_before();
      mbar_arrive(p_full(wg));
    }
    const bool fin = ok && (n_items == 0 ||
                            mbar_wait(acc_done, 0, abort_flag, p.err, p.timeout_ns));
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const size_t orow = (static_cast<size_t>(b * p.Hkv + hkv) * p.Nk + kr) * D;
      const bool valid = kr < p.Nk;
      const int c0 = wg * (D / 2);                     // this warpgroup's half of the columns
      if (n_items == 0) {
        if (valid) {
          store_zero_cols(p.dv + orow, c0, D / 2);
          store_zero_cols(p.dk + orow, c0, D / 2);
        }
      } else {
        store_cols_bf16(tmem + lane_base + 256, c0, D / 2, 1.f, p.dv + orow, valid, p.err);
        store_cols_bf16(tmem + lane_base + 256 + D, c0, D / 2, p.scale, p.dk + orow, valid,
                        p.err);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ
// Two softmax warpgroups over the same 128 query rows: warpgroup w takes keys
// 64 w .. 64 w + 63 of each key tile (columns 64 w .. of S and 128 + 64 w .. of
// dP) and writes its dS there as 32 columns of bf16 pairs; dQ takes each
// half's keys as soon as its warpgroup has released it.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work: query tile i of (b, h); CTAs from the last query tile down, so under the
  // causal mask the heaviest tiles (the most key tiles) start first
  const int n_qt = (p.Nq + kBM - 1) / kBM;
  const int nbh = p.B * p.Hq;
  const int i = n_qt - 1 - static_cast<int>(blockIdx.x) / nbh;
  const int bh = static_cast<int>(blockIdx.x) - (n_qt - 1 - i) * nbh;   // b * Hq + h
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int hkv = h / (p.Hq / p.Hkv);
  const int off = p.Nk - p.Nq;
  int n_kt = (p.Nk + kBM - 1) / kBM;
  if (p.causal) {
    const int last_row = min(i * kBM + kBM - 1, p.Nq - 1);
    n_kt = min(n_kt, (last_row + off) / kBM + 1);
  }

  auto bar = [&](int x) -> uint32_t { return sbase + L::kBarOff + 8 * x; };
  const uint32_t q_full = bar(0);
  auto kv_full = [&](int s) { return bar(1 + s); };
  auto kv_empty = [&](int s) { return bar(3 + s); };
  auto s_full = [&](int hh) { return bar(5 + hh); };
  auto ds_full = [&](int hh) { return bar(7 + hh); };
  const uint32_t acc_done = bar(9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const uint32_t q_smem = sbase + L::kFixOff;
  const uint32_t do_smem = sbase + L::kFixOff + L::kTileBytes;
  auto k_smem = [&](int s) { return sbase + L::kRingOff + (2 * s) * L::kTileBytes; };
  auto v_smem = [&](int s) { return sbase + L::kRingOff + (2 * s + 1) * L::kTileBytes; };

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(ds_full(s), kBM);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: [0,128) S then dS (warpgroup w's bf16 pairs in [64w, 64w+32));
  // [128,256) dP; [256,256+D) dQ

  if (warp == kProducerWarp) {
    if (lane == 0 && n_kt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(q_full, 2 * L::kTileBytes);
      for (int ch = 0; ch < L::kChunks; ++ch) {
        tma_load_3d(q_smem + ch * L::kChunkBytes, &tmQ, q_full, ch * 64, i * kBM, bh);
        tma_load_3d(do_smem + ch * L::kChunkBytes, &tmdO, q_full, ch * 64, i * kBM, bh);
      }
      const int z_kv = b * p.Hkv + hkv;
      int jt = 0;
      for (; jt < n_kt; ++jt) {
        const int s = jt & 1;
        if (!mbar_wait(kv_empty(s), ((jt >> 1) & 1) ^ 1, abort_flag, p.err, p.timeout_ns)) break;
        mbar_arrive_expect_tx(kv_full(s), 2 * L::kTileBytes);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(k_smem(s) + ch * L::kChunkBytes, &tmK, kv_full(s), ch * 64, jt * kBM, z_kv);
          tma_load_3d(v_smem(s) + ch * L::kChunkBytes, &tmV, kv_full(s), ch * 64, jt * kBM, z_kv);
        }
      }
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort, p.err, p.timeout_ns);
      for (int s = 0; s < 2 && s < jt; ++s) {
        const int last = s + ((jt - 1 - s) / 2) * 2;
        mbar_wait(kv_full(s), (last >> 1) & 1, &no_abort, p.err, p.timeout_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    const bool leader = elect_one();
    auto wait = [&](uint32_t br, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(br, parity, abort_flag, p.err, p.timeout_ns));
    };
    const uint64_t q_desc = smem_desc_sw128(q_smem, 16, 1024);
    const uint64_t do_desc = smem_desc_sw128(do_smem, 16, 1024);
    bool ok = n_kt == 0 || wait(q_full, 0);
    for (int jt = 0; ok && jt < n_kt; ++jt) {
      const int s = jt & 1;
      ok = wait(kv_full(s), (jt >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint64_t kd = smem_desc_sw128(k_smem(s), 16, 1024);
      const uint64_t vd = smem_desc_sw128(v_smem(s), 16, 1024);
      if (leader) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          mma_rows_x_half<D>(tmem + kHalfN * hh, q_desc, kd, kHalfN * hh);          // S
          mma_rows_x_half<D>(tmem + 128 + kHalfN * hh, do_desc, vd, kHalfN * hh);   // dP
          tc_commit(s_full(hh));
        }
      }
      const uint64_t k_mn = smem_desc_sw128(k_smem(s), L::kChunkBytes, 1024);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        ok = wait(ds_full(hh), jt & 1);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS K_j over this half's keys (K_j read MN-major: D contiguous)
        if (leader)
          mma_half_x_tile<D>(tmem + 256, tmem + kHalfN * hh, k_mn, kHalfN * hh, jt > 0 || hh > 0);
      }
      if (!ok) break;
      if (leader) tc_commit(kv_empty(s));
    }
    if (leader) tc_commit(acc_done);
    volatile int no_abort = 0;
    mbar_wait(acc_done, 0, &no_abort, p.err, p.timeout_ns);
  } else {
    const int wg = warp >> 2;                           // keys 64 wg .. 64 wg + 63
    const int r = (warp & 3) * 32 + lane;
    const int row = i * kBM + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + kHalfN * wg;
    const uint32_t tP = tmem + lane_base + 128 + kHalfN * wg;
    const size_t grow = static_cast<size_t>(bh) * p.Nq + row;
    float lse2 = INFINITY, dl = 0.f;
    if (row < p.Nq) {
      lse2 = __ldg(p.lse + grow) * kLog2e;
      dl = __ldg(p.delta + grow);
    }
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t nl2 = f2_pack(-lse2, -lse2);
    const uint64_t dl2 = f2_pack(dl, dl);
    bool ok = true;
    for (int jt = 0; ok && jt < n_kt; ++jt) {
      const bool got = mbar_wait(s_full(wg), jt & 1, abort_flag, p.err, p.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kbase = jt * kBM + kHalfN * wg;        // first key of this half
      const bool need_mask =
          (kbase + kHalfN > p.Nk) || (p.causal && kbase + kHalfN - 1 > i * kBM + off);
      int lim = p.Nk - 1 - kbase;
      if (p.causal) lim = min(lim, row + off - kbase);
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + 32 * c, sv, p.err);
        tmem_ld32(tP + 32 * c, dv, p.err);
        tmem_wait_ld(p.err);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2, nl2),
                    x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (need_mask) {
            if (32 * c + e > lim) p0 = 0.f;
            if (32 * c + e + 1 > lim) p1 = 0.f;
          }
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1),
                           f2_sub(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])),
                                  dl2)),
                    d0, d1);
          pk[e >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tS + 16 * c, pk, p.err);     // over columns already read
      }
      tmem_wait_st(p.err);
      tc_fence_before();
      mbar_arrive(ds_full(wg));
    }
    const bool fin = ok && (n_kt == 0 || mbar_wait(acc_done, 0, abort_flag, p.err, p.timeout_ns));
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      uint16_t* dst = p.dq + grow * D;
      const int c0 = wg * (D / 2);
      if (n_kt == 0) {
        if (row < p.Nq) store_zero_cols(dst, c0, D / 2);
      } else {
        store_cols_bf16(tmem + lane_base + 256, c0, D / 2, p.scale, dst, row < p.Nq, p.err);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// 3-D map over a contiguous [Z, N, D] bf16 tensor, box {64, 128, 1}, 128-byte swizzle.
int encode_tile_map(CUtensorMap* m, const void* base, int D, int N, int Z) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(Z)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                               static_cast<uint64_t>(N) * static_cast<uint64_t>(D) * 2};
  const uint32_t box[3] = {64, 128, 1};
  return encode_tensor_map_16bit(m, base, true, 3, dims, strides, box);
}

template <int D>
int launch_bwd_typed(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                     float* delta, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                     int causal, cudaStream_t stream, int device) {
  using L = BwdLayout<D>;
  static int attr_gen[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> g(mu);
    if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
    if (attr_gen[device] != cache_generation()) {
      cudaError_t e = cudaFuncSetAttribute(fa_bwd_dkdv_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           L::kSmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fa_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 L::kSmemBytes);
      if (e != cudaSuccess)
        return set_error(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      attr_gen[device] = cache_generation();
    }
  }
  BwdParams prm;
  prm.o = static_cast<const uint16_t*>(o);
  prm.dout = static_cast<const uint16_t*>(dout);
  prm.lse = lse;
  prm.delta = delta;
  prm.dq = static_cast<uint16_t*>(dq);
  prm.dk = static_cast<uint16_t*>(dk);
  prm.dv = static_cast<uint16_t*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal = causal ? 1 : 0;
  prm.scale = scale;
  prm.scale_log2 = scale * kLog2e;
  prm.err = device_error_word(device);
  prm.timeout_ns = kWaitLimitNs;
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");

  const long long rows = static_cast<long long>(B) * Hq * Nq;
  const int nsm = device_sm_count(device);
  if (nsm <= 0) return set_error(FA_ERR_CUDA, "cannot read the SM count of device %d", device);
  const int dgrid = static_cast<int>(std::min<long long>((rows + 7) / 8, 16LL * nsm));
  if (dgrid > 0)
    fa_bwd_delta_kernel<D><<<dgrid, 256, 0, stream>>>(prm.o, prm.dout, delta, rows);

  // A side with no rows (Nq == 0: dK = dV = 0; Nk == 0: dQ = 0) gets a copy of
  // the other side's maps, which its kernel then never reads.
  CUtensorMap tq, tk, tv, tdo;
  int rc;
  if (Nq > 0) {
    if ((rc = encode_tile_map(&tq, q, D, Nq, B * Hq)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tdo, dout, D, Nq, B * Hq)) != FA_OK) return rc;
  }
  if (Nk > 0) {
    if ((rc = encode_tile_map(&tk, k, D, Nk, B * Hkv)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&tv, v, D, Nk, B * Hkv)) != FA_OK) return rc;
  }
  if (Nq == 0 && Nk == 0) return FA_OK;
  if (Nq == 0) {
    tq = tk;
    tdo = tk;
  }
  if (Nk == 0) {
    tk = tq;
    tv = tq;
  }
  const long long kv_ctas = static_cast<long long>(B) * Hkv * ((Nk + kBM - 1) / kBM);
  const long long q_ctas = static_cast<long long>(B) * Hq * ((Nq + kBM - 1) / kBM);
  if (kv_ctas > 0x7fffffffLL || q_ctas > 0x7fffffffLL)
    return set_error(FA_ERR_UNSUPPORTED, "too many tiles");
  if (kv_ctas > 0)
    fa_bwd_dkdv_kernel<D><<<static_cast<unsigned>(kv_ctas), kThreads, L::kSmemBytes, stream>>>(
        tq, tk, tv, tdo, prm);
  if (q_ctas > 0)
    fa_bwd_dq_kernel<D><<<static_cast<unsigned>(q_ctas), kThreads, L::kSmemBytes, stream>>>(
        tq, tk, tv, tdo, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "fa_bwd launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace

int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, float* delta, int B, int Hq,
               int Hkv, int Nq, int Nk, int D, float scale, int causal, cudaStream_t stream,
               int device) {
  if (D == 128)
    return launch_bwd_typed<128>(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk,
                                 scale, causal, stream, device);
  if (D == 64)
    return launch_bwd_typed<64>(q, k, v, o, lse, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk,
                                scale, causal, stream, device);
  return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
}

}  // namespace fa
