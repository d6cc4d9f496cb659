// FP8 (E4M3) exact tiled attention forward for sm_100a, and the quantiser that
// prepares its inputs.
//
// Method: the blockwise online softmax of unite.ai, "Flash Attention:
// Revolutionizing Transformer Efficiency", section "Implementation Details",
// with the FP8 inputs, block quantisation and incoherent processing that the
// page's section "Flash Attention-3" lists among that version's additions.
//
// Quantiser (fa_quant_kernel): one CTA per 128-row group of a [Z, N, D] bf16
// slice, eight warps of 16 rows, each row spread over a warp (D / 32 values per
// lane, loads and stores coalesced).  Optionally every row is first rotated by
// diag(signs) H / sqrt(D) (H the Walsh-Hadamard matrix): one fp32 product per
// element, then the fast Walsh-Hadamard transform in fp32, butterfly stages in
// increasing bit order (the bits below log2(D / 32) inside a lane, the others
// across lanes by shuffles).  The group's amax gives r = 448 / amax and the
// stored scale amax / 448 (IEEE-rounded divisions), and each code is the
// round-to-nearest-even, saturating E4M3 conversion of the fp32 product x * r.
// Whole-slice groups (V) take three launches: the groups' amaxes are combined
// by an atomic maximum into the slice's scale slot, the codes are written with
// that amax, and a last kernel turns the amaxes into scales.
//
// Attention (fa_fwd_fp8_kernel): the structure of the bf16 kernel (persistent
// CTAs walking (pair of 128-row query tiles, sequence, head) items in snake
// order; warps 0-7 softmax, one per query tile and TMEM lane quarter; warp 8
// TMA producer; warp 9 MMA issuer; warps 10-11 idle; K/V ring and barrier
// phases running on across items), with D = 128 one-byte codes per row, so a
// Q, K or V tile is 16 KB, one 128-byte swizzle atom wide, and the ring holds
// ten of them.  S = Q K^T and O += P V are tcgen05 kind::f8f6f4 MMAs (32 K
// elements per instruction, fp32 accumulation in TMEM).  The softmax converts
// raw scores to scaled log2 units with the tile's factor
// scale * log2(e) * q_scale * k_scale_j and writes P back over the first 32
// columns of its S tile as E4M3 (four per column), offset so that the row's
// reference maximum maps to 2^6: p = 2^(x - m_ref + 6).  With a lazy-rescale
// threshold of 2.5 every p is at most 2^8.5 < 448 (the reference moves, and O is
// rescaled, only when a tile's maximum exceeds it by more than 2.5), and entries
// down to 2^-12 of the reference stay normal E4M3 numbers (below that the
// subnormal spacing 2^-9 is at most 2^-15 of the row's largest p).  The row sum
// L is taken over the unrounded p; O is multiplied by v_scale / L at the end
// and LSE removes the offset.
#include <algorithm>
#include <cfloat>
#include <cstdio>
#include <mutex>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {
namespace {

// ---------------------------------------------------------------- quantiser
constexpr int kQuantRows = 128;          // rows per group (a query or key tile)
constexpr int kQuantThreads = 256;       // 8 warps x 16 rows
constexpr int kQuantRowsPerWarp = 16;
enum : int { kQuantGroups = 0, kQuantSliceAmax = 1, kQuantSlice = 2 };

// Fast Walsh-Hadamard transform of one row held by a warp, E = D / 32
// consecutive elements per lane (lane l holds l E .. l E + E - 1).  Each stage
// b maps the pair (i, i + 2^b) with bit b of i clear to (x_i + x_j, x_i - x_j).
template <int E>
__device__ __forceinline__ void fwht_row(float (&v)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (!(e & h)) {
        const float a = v[e], c = v[e | h];
        v[e] = __fadd_rn(a, c);
        v[e | h] = __fsub_rn(a, c);
      }
#pragma unroll
  for (int lb = 1; lb < 32; lb <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], lb);
      v[e] = (lane & lb) ? __fsub_rn(other, v[e]) : __fadd_rn(v[e], other);
    }
}

// The same transform with a row held by a lane pair, 64 consecutive elements
// per lane (lane 2k + h holds 64 h .. 64 h + 63 of its row): the stages of
// strides 1 to 32 stay in registers and only the stride-64 stage crosses
// lanes.  The stages run in the same order with the same additions as
// fwht_row, so every result is bit-identical.
__device__ __forceinline__ void fwht_row_pair(float (&v)[64], int lane) {
#pragma unroll
  for (int h = 1; h < 64; h <<= 1)
#pragma unroll
    for (int e = 0; e < 64; ++e)
      if (!(e & h)) {
        const float a = v[e], c = v[e | h];
        v[e] = __fadd_rn(a, c);
        v[e | h] = __fsub_rn(a, c);
      }
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const float other = __shfl_xor_sync(0xffffffffu, v[e], 1);
    v[e] = (lane & 1) ? __fsub_rn(other, v[e]) : __fadd_rn(v[e], other);
  }
}

// Byte offset of 16-byte chunk `c` (0-15) of row `r` in a warp's staging area
// of 16 rows x 256 bytes: chunks XOR-swizzled by the row within each 128-byte
// half, so a lane pair per row reads and writes without bank conflicts beyond
// the four wavefronts a 512-byte access needs.
__device__ __forceinline__ uint32_t qstage_off(int r, int c) {
  return static_cast<uint32_t>(r * 256 + (c & 8) * 16 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D, bool ROT, int MODE>
__global__ void __launch_bounds__(kQuantThreads, 3)
    fa_quant_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                    float* __restrict__ scales, const float* __restrict__ signs, int N,
                    int groups) {
  constexpr int E = D / 32;
  __shared__ float warp_amax[kQuantThreads / 32];
  if constexpr (D == 128) {
    // Each warp's 16 rows (4 KB of bf16, contiguous in global memory) pass
    // through shared memory: coalesced 16-byte global loads and stores, and a
    // lane pair per row in registers.
    __shared__ __align__(16) uint8_t stage_all[kQuantThreads / 32][16 * 256];
    __shared__ float mult_sm[128];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int half = lane & 1;
    const int rw = lane >> 1;                    // this lane's row within the warp's 16
    const int g = blockIdx.x;
    const int z = blockIdx.y;
    const size_t slice = static_cast<size_t>(z) * N * D;
    const int wrow0 = g * kQuantRows + warp * kQuantRowsPerWarp;
    const uint32_t stage = smem_u32(stage_all[warp]);
    if constexpr (ROT) {
      if (threadIdx.x < 128)
        mult_sm[threadIdx.x] = __fmul_rn(__ldg(signs + threadIdx.x), 0.0883883476483184405f);
    }
    // global -> shared: instruction k moves 512 contiguous bytes (rows 2k, 2k + 1)
    const uint4* gsrc = reinterpret_cast<const uint4*>(x + slice + static_cast<size_t>(wrow0) * D);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int ci = k * 32 + lane;              // 16-byte chunk of the warp's 4 KB
      const int r = ci >> 4;
      const uint4 u = (wrow0 + r < N) ? __ldg(gsrc + ci) : make_uint4(0u, 0u, 0u, 0u);
      st_shared_v4(stage + qstage_off(r, ci & 15), u.x, u.y, u.z, u.w);
    }
    __syncwarp();
    float v[64];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t u[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                   : "r"(stage + qstage_off(rw, half * 8 + k)));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[8 * k + 2 * q] = __uint_as_float(u[q] << 16);
        v[8 * k + 2 * q + 1] = __uint_as_float(u[q] & 0xffff0000u);
      }
    }
    if constexpr (ROT) {
      __syncthreads();                           // mult_sm is written
#pragma unroll
      for (int e = 0; e < 64; ++e) v[e] = __fmul_rn(v[e], mult_sm[half * 64 + e]);
      fwht_row_pair(v, lane);
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 64; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) warp_amax[warp] = amax;
    __syncthreads();
    amax = warp_amax[0];
#pragma unroll
    for (int w2 = 1; w2 < kQuantThreads / 32; ++w2) amax = fmaxf(amax, warp_amax[w2]);
    if constexpr (MODE == kQuantSliceAmax) {
      if (threadIdx.x == 0)
        atomicMax(reinterpret_cast<unsigned int*>(scales) + z, __float_as_uint(amax));
      return;
    } else {
      if constexpr (MODE == kQuantSlice)
        amax = __uint_as_float(*reinterpret_cast<const volatile unsigned int*>(scales + z));
      const float rr = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
      if (MODE == kQuantGroups && threadIdx.x == 0)
        scales[static_cast<size_t>(z) * groups + g] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
      // codes -> shared (row rw's 128 code bytes at rw * 128, swizzled like the
      // input's halves), then shared -> global, 512 contiguous bytes per instruction
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t c4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = 16 * k + 4 * q;
          c4[q] = pack_e4m3x4(__fmul_rn(v[e], rr), __fmul_rn(v[e + 1], rr),
                              __fmul_rn(v[e + 2], rr), __fmul_rn(v[e + 3], rr));
        }
        const int cc = half * 4 + k;             // 16-byte chunk of the 128-byte code row
        st_shared_v4(stage + static_cast<uint32_t>(rw * 128 + ((cc ^ (rw & 7)) << 4)), c4[0],
                     c4[1], c4[2], c4[3]);
      }
      __syncwarp();
      uint4* gdst = reinterpret_cast<uint4*>(codes + slice + static_cast<size_t>(wrow0) * D);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int ci = k * 32 + lane;            // 16-byte chunk of the warp's 2 KB of codes
        const int r = ci >> 3;
        if (wrow0 + r < N) {
          uint32_t u[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                       : "r"(stage + static_cast<uint32_t>(r * 128 + (((ci & 7) ^ (r & 7)) << 4))));
          gdst[ci] = make_uint4(u[0], u[1], u[2], u[3]);
        }
      }
    }
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int z = blockIdx.y;
  const size_t slice = static_cast<size_t>(z) * N * D;
  const int row0 = g * kQuantRows + warp * kQuantRowsPerWarp;

  float mult[E];
  if constexpr (ROT) {
    const float c = D == 128 ? 0.0883883476483184405f : 0.125f;   // fp32(1 / sqrt(D))
#pragma unroll
    for (int e = 0; e < E; ++e) mult[e] = __fmul_rn(__ldg(signs + lane * E + e), c);
  }
  // all 16 rows' loads are issued before any arithmetic, so they are in flight
  // together (rows past N read as zero and are not stored)
  uint32_t w[kQuantRowsPerWarp][E / 2];
#pragma unroll
  for (int i = 0; i < kQuantRowsPerWarp; ++i) {
    const int row = row0 + i;                    // warp-uniform
    const uint16_t* src = x + slice + static_cast<size_t>(row) * D + lane * E;
    if constexpr (E == 4) {
      uint2 u = make_uint2(0u, 0u);
      if (row < N) u = __ldg(reinterpret_cast<const uint2*>(src));
      w[i][0] = u.x;
      w[i][1] = u.y;
    } else {
      w[i][0] = row < N ? __ldg(reinterpret_cast<const uint32_t*>(src)) : 0u;
    }
  }
  float v[kQuantRowsPerWarp][E];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kQuantRowsPerWarp; ++i) {
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      v[i][2 * e] = __uint_as_float(w[i][e] << 16);
      v[i][2 * e + 1] = __uint_as_float(w[i][e] & 0xffff0000u);
    }
    if constexpr (ROT) {
#pragma unroll
      for (int e = 0; e < E; ++e) v[i][e] = __fmul_rn(v[i][e], mult[e]);
      fwht_row<E>(v[i], lane);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) warp_amax[warp] = amax;
  __syncthreads();
  amax = warp_amax[0];
#pragma unroll
  for (int w2 = 1; w2 < kQuantThreads / 32; ++w2) amax = fmaxf(amax, warp_amax[w2]);

  if constexpr (MODE == kQuantSliceAmax) {
    // non-negative floats order like their bit patterns
    if (threadIdx.x == 0)
      atomicMax(reinterpret_cast<unsigned int*>(scales) + z, __float_as_uint(amax));
    return;
  } else {
    if constexpr (MODE == kQuantSlice)
      amax = __uint_as_float(*reinterpret_cast<const volatile unsigned int*>(scales + z));
    const float r = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
    if (MODE == kQuantGroups && threadIdx.x == 0)
      scales[static_cast<size_t>(z) * groups + g] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
    for (int i = 0; i < kQuantRowsPerWarp; ++i) {
      const int row = row0 + i;
      if (row < N) {
        uint8_t* dst = codes + slice + static_cast<size_t>(row) * D + lane * E;
        if constexpr (E == 4)
          *reinterpret_cast<uint32_t*>(dst) =
              pack_e4m3x4(__fmul_rn(v[i][0], r), __fmul_rn(v[i][1], r), __fmul_rn(v[i][2], r),
                          __fmul_rn(v[i][3], r));
        else
          *reinterpret_cast<uint16_t*>(dst) =
              pack_e4m3x2(__fmul_rn(v[i][0], r), __fmul_rn(v[i][1], r));
      }
    }
  }
}

// Slice amax -> scale (amax / 448, or 1 for an all-zero slice).
__global__ void fa_quant_finalize_kernel(float* scales, int Z) {
  const int z = blockIdx.x * blockDim.x + threadIdx.x;
  if (z < Z) {
    const float a = scales[z];
    scales[z] = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
  }
}

template <int D, bool ROT>
int launch_quant_typed(const void* x, void* codes, float* scales, int Z, int N, int group_rows,
                       const float* signs, cudaStream_t stream) {
  const int groups = (N + kQuantRows - 1) / kQuantRows;
  const dim3 grid(static_cast<unsigned>(groups), static_cast<unsigned>(Z));
  const auto* xs = static_cast<const uint16_t*>(x);
  auto* cs = static_cast<uint8_t*>(codes);
  if (group_rows == kQuantRows) {
    if (groups > 0)
      fa_quant_kernel<D, ROT, kQuantGroups><<<grid, kQuantThreads, 0, stream>>>(
          xs, cs, scales, signs, N, groups);
  } else {
    // an empty slice keeps amax 0 and so gets scale 1
    cudaError_t e = cudaMemsetAsync(scales, 0, static_cast<size_t>(Z) * sizeof(float), stream);
    if (e != cudaSuccess)
      return set_error(FA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    if (groups > 0) {
      fa_quant_kernel<D, ROT, kQuantSliceAmax><<<grid, kQuantThreads, 0, stream>>>(
          xs, cs, scales, signs, N, groups);
      fa_quant_kernel<D, ROT, kQuantSlice><<<grid, kQuantThreads, 0, stream>>>(
          xs, cs, scales, signs, N, groups);
    }
    fa_quant_finalize_kernel<<<(Z + 255) / 256, 256, 0, stream>>>(scales, Z);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "fa_quantize_e4m3 launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

// ---------------------------------------------------------------- attention
constexpr int kBM = 128;            // query rows per tile = TMEM lanes
constexpr int kBN = 128;            // keys per tile
constexpr int kD = 128;             // head dimension (one byte per element)
constexpr int kTile = kBM * kD;     // bytes of a Q, K or V tile
constexpr int kSlots = 10;          // K/V ring slots
constexpr float kTau = 2.5f;        // lazy-rescale threshold (log2 units)
constexpr float kPOff = 6.f;        // p = 2^(x - m_ref + kPOff)
constexpr float kPScale = 64.f;     // 2^kPOff
constexpr int kThreads = 384;
#ifndef FA_FP8_HALF_EXP
#define FA_FP8_HALF_EXP 0
#endif
// 1: the exponentials of P in f16 pairs (ex2.approx.f16x2), converted straight
// to E4M3; 0: one fp32 exponential per element.
constexpr bool kHalfExp = FA_FP8_HALF_EXP != 0;
constexpr uint32_t kF16x2Off = 0x54005400u;   // (64, 64) in f16: 2^kPOff
constexpr uint32_t kRegsControl = 72;
constexpr uint32_t kRegsSoftmax = 216;
static_assert(kRegsControl * 128 + kRegsSoftmax * 256 <= 384 * 168, "register split");
static_assert(448.f > 362.1f, "2^(kPOff + kTau) must stay below E4M3's largest value");

struct Fp8Layout {
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTile;
  static constexpr int kBarOff = kKVOff + kSlots * kTile;
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 4 + 2 + 1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem address, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;   // + slack for 1024-byte alignment
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Fp8Params {
  void* o;
  float* lse;
  const float* q_scale;   // [B * Hq, nqg]
  const float* k_scale;   // [B * Hkv, nkg]
  const float* v_scale;   // [B * Hkv]
  int B, Hq, Hkv, Nq, Nk;
  int nqg, nkg;           // 128-row scale groups per (sequence, head)
  int num_mpairs;
  int num_items;          // num_mpairs * B * Hq, heaviest first when causal
  int causal;
  float scale_log2;       // scale * log2(e)
  int* err;
  uint64_t timeout_ns;
};

__device__ __forceinline__ int kv_tiles(int first_row, int Nq, int Nk, int causal) {
  if (first_row >= Nq) return 0;
  const int nk_tiles = (Nk + kBN - 1) / kBN;
  if (!causal) return nk_tiles;
  const int last_row = min(first_row + kBM - 1, Nq - 1);
  return min(nk_tiles, (last_row + (Nk - Nq)) / kBN + 1);
}

struct Fp8Item {
  int bh, b, h, hkv, q_row0, n0, n1;
};

// Item r * C + (r odd ? C - 1 - cta : cta) of round r: the list runs over tile
// pairs (heaviest first when causal), then sequences and heads.
__device__ __forceinline__ bool fp8_item(const Fp8Params& p, int cta, int C, int r, Fp8Item& it) {
  const int i = r * C + ((r & 1) ? C - 1 - cta : cta);
  if (i >= p.num_items) return false;
  const int BH = p.B * p.Hq;
  const int mrev = i / BH;
  it.bh = i - mrev * BH;
  it.b = it.bh / p.Hq;
  it.h = it.bh - it.b * p.Hq;
  it.hkv = it.h / (p.Hq / p.Hkv);
  const int m = p.causal ? (p.num_mpairs - 1 - mrev) : mrev;
  it.q_row0 = m * 2 * kBM;
  it.n0 = kv_tiles(it.q_row0, p.Nq, p.Nk, p.causal);
  it.n1 = kv_tiles(it.q_row0 + kBM, p.Nq, p.Nk, p.causal);
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Fp8Params p) {
  using L = Fp8Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int C = gridDim.x;
  const int cta = blockIdx.x;

  auto bar = [&](int i) -> uint32_t { return sbase + L::kBarOff + 8 * i; };
  auto q_full = [&](int t) { return bar(t); };
  auto kv_full = [&](int s) { return bar(2 + s); };
  auto kv_empty = [&](int s) { return bar(2 + kSlots + s); };
  auto s_full = [&](int t) { return bar(2 + 2 * kSlots + t); };
  auto p_half = [&](int t, int h) { return bar(4 + 2 * kSlots + 2 * t + h); };
  auto o_full = [&](int t) { return bar(8 + 2 * kSlots + t); };
  const uint32_t mma_done = bar(10 + 2 * kSlots);
  const uint32_t q_empty = bar(11 + 2 * kSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (tid == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_half(t, 0), kBM);
      mbar_init(p_half(t, 1), kBM);
      mbar_init(o_full(t), 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(q_empty, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == 8) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int pos = 0, items = 0;
        bool ok = true;
        Fp8Item it;
        for (int r = 0; ok && fp8_item(p, cta, C, r, it); ++r) {
          const int n_max = max(it.n0, it.n1);
          if (n_max == 0) continue;
          if (items > 0 && !mbar_wait(q_empty, (items - 1) & 1, abort_flag, p.err, p.timeout_ns))
            break;
          for (int t = 0; t < 2; ++t) {   // [B * Hq, Nq, 128] bytes: box {128, 128 rows, 1}
            mbar_arrive_expect_tx(q_full(t), kTile);
            tma_load_3d(sbase + L::kQOff + t * kTile, &tmQ, q_full(t), 0, it.q_row0 + t * kBM,
                        it.bh);
          }
          ++items;
          const int kv_z = it.b * p.Hkv + it.hkv;
          for (int j = 0; j < n_max && ok; ++j) {
            for (int w = 0; w < 2; ++w, ++pos) {
              const int slot = pos % kSlots;
              const uint32_t ph = (pos / kSlots) & 1;
              if (!mbar_wait(kv_empty(slot), ph ^ 1, abort_flag, p.err, p.timeout_ns)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(kv_full(slot), kTile);
              const void* tm = w ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmK);
              tma_load_3d(sbase + L::kKVOff + slot * kTile, tm, kv_full(slot), 0, j * kBN, kv_z);
            }
          }
        }
        // Every issued copy must land before the CTA may exit (also on abort).
        volatile int no_abort = 0;
        if (items > 0)
          for (int t = 0; t < 2; ++t)
            mbar_wait(q_full(t), (items - 1) & 1, &no_abort, p.err, p.timeout_ns);
        for (int sl = 0; sl < kSlots && sl < pos; ++sl) {
          const int last = sl + ((pos - 1 - sl) / kSlots) * kSlots;
          mbar_wait(kv_full(sl), (last / kSlots) & 1, &no_abort, p.err, p.timeout_ns);
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      const bool leader = elect_one();
      constexpr uint32_t idesc_s = idesc_e4m3(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_e4m3(kBM, kD, true);
      auto slot_of = [&](int pos) { return pos % kSlots; };
      auto phase_of = [&](int pos) { return static_cast<uint32_t>((pos / kSlots) & 1); };
      auto wait = [&](uint32_t b, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, p.err, p.timeout_ns));
      };
      auto commit = [&](uint32_t b) {
        if (leader) tc_commit(b);
      };
      // K-major Q and K (rows of 128 one-byte head dims); V MN-major (a key's
      // 128 head dims contiguous).  One swizzle atom spans the head dimension,
      // so a K step of 32 elements moves the start address by 32 bytes.
      const uint64_t desc_q0 = smem_desc_sw128(sbase + L::kQOff, 16, 1024);
      const uint64_t desc_q1 = smem_desc_sw128(sbase + L::kQOff + kTile, 16, 1024);
      const uint64_t desc_k = smem_desc_sw128(sbase + L::kKVOff, 16, 1024);
      const uint64_t desc_v = smem_desc_sw128(sbase + L::kKVOff, kTile, 1024);
      auto issue_s = [&](int t, int slot) {
        const uint64_t a0 = t ? desc_q1 : desc_q0;
        const uint64_t b0 = desc_k + static_cast<uint64_t>((slot * kTile) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kD / 32; ++kk)
            mma_ss_f8(tmem + t * 128, a0 + 2 * kk, b0 + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
          tc_commit(s_full(t));
        }
      };
      // O_t += P_t V over keys [64 h, 64 h + 64): P from TMEM (E4M3, four per
      // column), V rows of 32 keys = 4096 bytes per K step.
      auto issue_pv_half = [&](int t, int slot, int h, bool accumulate) {
        const uint64_t b0 = desc_v + static_cast<uint64_t>((slot * kTile) >> 4);
        if (leader) {
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int kk = 2 * h + k2;
            mma_ts_f8(tmem + 256 + t * kD, tmem + t * 128 + kk * 8,
                      b0 + static_cast<uint64_t>((kk * 32 * kD) >> 4), idesc_pv,
                      (accumulate || kk > 0) ? 1u : 0u);
          }
        }
      };
      bool ok = true;
      int pos = 0, items = 0;
      int tiles[2] = {0, 0};
      Fp8Item it;
      for (int r = 0; ok && fp8_item(p, cta, C, r, it); ++r) {
        const int n_max = max(it.n0, it.n1);
        if (n_max == 0) continue;
        ok = wait(q_full(0), items & 1);
        if (ok) ok = wait(q_full(1), items & 1);
        if (ok) ok = wait(kv_full(slot_of(pos)), phase_of(pos));
        if (!ok) break;
        ++items;
        tc_fence_after();
        if (it.n0 > 0) issue_s(0, slot_of(pos));
        if (it.n1 > 0) issue_s(1, slot_of(pos));
        commit(kv_empty(slot_of(pos)));
        if (n_max == 1) commit(q_empty);
        for (int j = 0; j < n_max && ok; ++j) {
          const int vpos = pos + 2 * j + 1;
          const int kpos = pos + 2 * j + 2;
          const bool has_next = j + 1 < n_max;
          ok = wait(kv_full(slot_of(vpos)), phase_of(vpos));
          bool k_ready = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int nt = t ? it.n1 : it.n0;
            if (!ok || j >= nt) continue;
            const uint32_t par = static_cast<uint32_t>((tiles[t] + j) & 1);
            ok = wait(p_half(t, 0), par);
            if (!ok) continue;
            tc_fence_after();
            issue_pv_half(t, slot_of(vpos), 0, j > 0);
            ok = wait(p_half(t, 1), par);
            if (!ok) continue;
            tc_fence_after();
            issue_pv_half(t, slot_of(vpos), 1, true);
            if (j + 1 < nt) {
              if (!k_ready) {
                ok = wait(kv_full(slot_of(kpos)), phase_of(kpos));
                k_ready = true;
                if (!ok) continue;
                tc_fence_after();
              }
              issue_s(t, slot_of(kpos));
            } else {
              commit(o_full(t));
            }
          }
          if (!ok) break;
          if (j + 2 == n_max) commit(q_empty);
          commit(kv_empty(slot_of(vpos)));
          if (has_next) commit(kv_empty(slot_of(kpos)));
        }
        pos += 2 * n_max;
        tiles[0] += it.n0;
        tiles[1] += it.n1;
      }
      commit(mma_done);
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, p.err, p.timeout_ns);
    }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + 256 + t * kD;
    int tiles = 0, outs = 0;
    bool ok = true;
    Fp8Item it;
    for (int rr = 0; ok && fp8_item(p, cta, C, rr, it); ++rr) {
      const int row = it.q_row0 + t * kBM + r;
      const int n = t ? it.n1 : it.n0;
      const size_t row_index = static_cast<size_t>(it.bh) * p.Nq + row;
      uint16_t* o_row = reinterpret_cast<uint16_t*>(p.o) + row_index * kD;
      if (n == 0) {
        if (max(it.n0, it.n1) == 0 && row < p.Nq) {   // only reached when Nk == 0
          const uint4 zero = make_uint4(0, 0, 0, 0);
          for (int ch = 0; ch < kD / 8; ++ch) reinterpret_cast<uint4*>(o_row)[ch] = zero;
          if (p.lse) p.lse[row_index] = -INFINITY;
        }
        continue;
      }
      const int kvh = it.b * p.Hkv + it.hkv;
      const float q_s = __ldg(p.q_scale + static_cast<size_t>(it.bh) * p.nqg +
                              (it.q_row0 / kBM + t));
      const float v_s = __ldg(p.v_scale + kvh);
      const float* k_s = p.k_scale + static_cast<size_t>(kvh) * p.nkg;
      const float qc = p.scale_log2 * q_s;
      float m_used = -INFINITY;
      float l = 0.f;
      const int off = p.Nk - p.Nq;
      const int tile_first = it.q_row0 + t * kBM;
      for (int j = 0; j < n; ++j) {
        const float c = qc * __ldg(k_s + j);   // raw score -> scaled log2 units
        const bool got = mbar_wait(s_full(t), (tiles + j) & 1, abort_flag, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]), p.err);
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]), p.err);
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]), p.err);
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]), p.err);
        tmem_wait_ld(p.err);
        const int kbase = j * kBN;
        const bool need_mask =
            (kbase + kBN > p.Nk) || (p.causal && kbase + kBN - 1 > tile_first + off);
        if (need_mask) {
          int lim = p.Nk - 1 - kbase;
          if (p.causal) lim = min(lim, row + off - kbase);
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > lim) s[e] = __float_as_uint(-INFINITY);
        }
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = __uint_as_float(s[k]);
#pragma unroll
        for (int e = 8; e + 16 <= 128; e += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            acc[k] = fmax3(acc[k], __uint_as_float(s[e + k]), __uint_as_float(s[e + 8 + k]));
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = fmaxf(acc[k], __uint_as_float(s[120 + k]));
        const float mx = fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]),
                               fmaxf(acc[6], acc[7]));
        const float m_tile = mx * c;
        const bool move = m_tile > m_used + kTau;
        float alpha = 1.f;
        if (move) {
          alpha = ex2(m_used - m_tile);
          l *= alpha;
          m_used = m_tile;
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
          for (int cc = 0; cc < kD / 32; ++cc) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * cc, ov, p.err);
            tmem_wait_ld(p.err);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + 32 * cc, ov, p.err);
          }
        }
        // the half-precision variant exponentiates x - m_ref (small for the
        // entries that matter, so f16 keeps them accurate) and applies the
        // 2^kPOff offset as an exact f16 product; its L then has no offset
        const float neg_m = (m_used == -INFINITY) ? 0.f : (kHalfExp ? 0.f : kPOff) - m_used;
        const uint64_t c2 = f2_pack(c, c);
        const uint64_t nm2 = f2_pack(neg_m, neg_m);
        uint64_t sum2[4] = {0, 0, 0, 0};
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {          // 32 keys -> 8 TMEM columns of 4 codes
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int k0 = 32 * cq + 4 * e;
            float x0, x1, x2, x3;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])), c2,
                             nm2), x0, x1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[k0 + 2]), __uint_as_float(s[k0 + 3])), c2,
                             nm2), x2, x3);
            if constexpr (kHalfExp) {
              // exponent pairs in f16, two exponentials per MUFU instruction
              const uint32_t h01 = ex2_f16x2(pack_f16x2(x0, x1));
              const uint32_t h23 = ex2_f16x2(pack_f16x2(x2, x3));
              float p0, p1, p2, p3;
              unpack_f16x2(h01, p0, p1);
              unpack_f16x2(h23, p2, p3);
              sum2[e & 3] = f2_add(sum2[e & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
              pk[e] = static_cast<uint32_t>(e4m3x2_from_f16x2(mul_f16x2(h01, kF16x2Off))) |
                      (static_cast<uint32_t>(e4m3x2_from_f16x2(mul_f16x2(h23, kF16x2Off)))
                       << 16);
            } else {
              const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
              sum2[e & 3] = f2_add(sum2[e & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
              pk[e] = pack_e4m3x4(p0, p1, p2, p3);
            }
          }
          tmem_st8(tS + 8 * cq, pk, p.err);
          if (cq == 1) {                           // keys 0-63 of P are in place
            tmem_wait_st(p.err);
            tc_fence_before();
            mbar_arrive(p_half(t, 0));
          }
        }
        float sa, sb;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sa, sb);
        l += sa + sb;
        tmem_wait_st(p.err);
        tc_fence_before();
        mbar_arrive(p_half(t, 1));
      }
      tiles += n;
      const bool fin = ok && mbar_wait(o_full(t), outs & 1, abort_flag, p.err, p.timeout_ns);
      ++outs;
      if (!__all_sync(0xffffffffu, fin)) {
        ok = false;
      } else {
        tc_fence_after();
        const float l_p = kHalfExp ? l * kPScale : l;   // the sum of the p that P holds
        const float inv = l > 0.f ? v_s / l_p : 0.f;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * cc, ov, p.err);
          tmem_wait_ld(p.err);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv,
                                __uint_as_float(ov[2 * e + 1]) * inv);
          if (row < p.Nq) {
            uint4* dst = reinterpret_cast<uint4*>(o_row + 32 * cc);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (p.lse && row < p.Nq)
          p.lse[row_index] =
              l > 0.f ? (m_used - (kHalfExp ? 0.f : kPOff) + __log2f(l)) * 0.69314718055994530942f
                      : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [Z, N, 128] one-byte codes, box {128, 128 rows, 1}, 128-byte swizzle.
int encode_codes(CUtensorMap* m, const void* base, int N, int Z) {
  const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(Z)};
  const uint64_t strides[2] = {static_cast<uint64_t>(kD),
                               static_cast<uint64_t>(N) * static_cast<uint64_t>(kD)};
  const uint32_t box[3] = {static_cast<uint32_t>(kD), static_cast<uint32_t>(kBM), 1};
  return encode_tensor_map_u8(m, base, 3, dims, strides, box);
}

}  // namespace

int launch_quantize_e4m3(const void* x, void* codes, float* scales, int Z, int N, int D,
                         int group_rows, const float* signs, cudaStream_t stream, int) {
  if (Z == 0) return FA_OK;
  if (D == 128)
    return signs ? launch_quant_typed<128, true>(x, codes, scales, Z, N, group_rows, signs, stream)
                 : launch_quant_typed<128, false>(x, codes, scales, Z, N, group_rows, signs,
                                                  stream);
  if (D == 64)
    return signs ? launch_quant_typed<64, true>(x, codes, scales, Z, N, group_rows, signs, stream)
                 : launch_quant_typed<64, false>(x, codes, scales, Z, N, group_rows, signs,
                                                 stream);
  return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
}

int launch_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                   const float* k_scale, const float* v_scale, void* o, float* lse, int B,
                   int Hq, int Hkv, int Nq, int Nk, float scale, int causal, cudaStream_t stream,
                   int device) {
  using L = Fp8Layout;
  static int attr_gen[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> g(mu);
    if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
    if (attr_gen[device] != cache_generation()) {
      cudaError_t e = cudaFuncSetAttribute(fa_fwd_fp8_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           L::kSmemBytes);
      if (e != cudaSuccess)
        return set_error(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      attr_gen[device] = cache_generation();
    }
  }
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = encode_codes(&tq, q8, Nq, B * Hq)) != FA_OK) return rc;
  if (Nk > 0) {
    if ((rc = encode_codes(&tk, k8, Nk, B * Hkv)) != FA_OK) return rc;
    if ((rc = encode_codes(&tv, v8, Nk, B * Hkv)) != FA_OK) return rc;
  } else {
    tk = tq;   // no key tile exists, so these maps are never read
    tv = tq;
  }
  Fp8Params prm;
  prm.o = o;
  prm.lse = lse;
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.v_scale = v_scale;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.nqg = (Nq + kBM - 1) / kBM;
  prm.nkg = (Nk + kBN - 1) / kBN;
  prm.num_mpairs = (Nq + 2 * kBM - 1) / (2 * kBM);
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = device_error_word(device);
  prm.timeout_ns = kWaitLimitNs;
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  const long long items = static_cast<long long>(prm.num_mpairs) * B * Hq;
  if (items > 0x7fffffffLL) return set_error(FA_ERR_UNSUPPORTED, "too many work items");
  prm.num_items = static_cast<int>(items);
  const int nsm = device_sm_count(device);
  if (nsm <= 0) return set_error(FA_ERR_CUDA, "cannot read the SM count of device %d", device);
  const int grid = static_cast<int>(std::min<long long>(items, nsm));
  if (grid == 0) return FA_OK;
  fa_fwd_fp8_kernel<<<static_cast<unsigned>(grid), kThreads, L::kSmemBytes, stream>>>(tq, tk, tv,
                                                                                       prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(FA_ERR_CUDA, "fa_fwd_fp8 launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace fa
