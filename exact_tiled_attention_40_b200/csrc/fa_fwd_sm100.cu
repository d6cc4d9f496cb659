// Exact tiled attention forward for sm_100a.
//
// Method: the blockwise online-softmax algorithm of unite.ai, "Flash Attention:
// Revolutionizing Transformer Efficiency", section "Implementation Details"
// (query blocks outer, key/value blocks inner, running row max M and row sum L),
// with the softmax decomposition and merge of section "The Mathematics of
// Flash Attention".  O is kept unnormalised and divided by L once at the end.
//
// Persistent: one CTA per SM walks a list of work items, each two 128-row query
// tiles (Q0, Q1) of one (sequence, head), streaming the 128-key K/V tiles of the
// matching KV head (GQA, devhandbook example 5) through a ring of shared-memory
// slots whose positions, like every barrier's phase, run on across items.
// Three instantiations share this code: dense [B, H, N, D] tensors, ragged
// batches packed as [total, H, D] with device row offsets, and ragged queries
// against keys/values in a 16-token page pool reached through a block table.
// Warp roles (384 threads, 3 warpgroups):
//   warps 0-3   softmax warpgroup for Q0   (thread r owns query row r = TMEM lane r)
//   warps 4-7   softmax warpgroup for Q1
//   warp  8     TMA producer: per item the Q tiles, then K_j, V_j into the slot ring
//   warp  9     TMEM allocator and MMA issuer (the warp runs the loop, one elected
//               lane issues the tcgen05 MMAs and commits)
//   warps 10-11 idle
// The control warpgroup (warps 8-11) hands registers to the softmax warpgroups
// (setmaxnreg): 72 and 216 per-thread registers over 128 + 256 threads equal
// the 384 x 168 the block is launched with.
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128) S0 = Q0 K^T  (its last 64 columns are reused for P0 as bf16 pairs)
//   [128,256) S1 = Q1 K^T  (P1 likewise)
//   [256,256+D) O0,  [256+D,256+2D) O1  -- the running unnormalised outputs
// Per key tile j the MMA thread issues, in order: PV0_j, S0_{j+1}, PV1_j, S1_{j+1},
// each PV in two halves of 64 keys that the softmax releases as it writes P.
// tcgen05 operations of one thread execute in issue order, so S_{j+1} never
// overwrites P_j before PV_j has read it, and the commit that publishes S_{j+1}
// also guarantees PV_j finished -- the softmax warpgroup may then rescale O in
// place before it releases P_{j+1}.  (The two query tiles' softmax phases
// settle into alternation: each one's MMAs run while the other computes.)
// The rescale is lazy: a row's reference maximum only moves when the new tile
// maximum exceeds it by more than 2^8, so P stays <= 256 and O is rescaled only
// on those rare tiles.  Exactness is unaffected: O and L share the reference.
#include <algorithm>
#include <cfloat>
#include <cstdio>
#include <mutex>

#include "fa_internal.h"
#include "ptx_sm100.cuh"
#include "../../include/fa.h"

namespace fa {
namespace {

constexpr int kBM = 128;       // query rows per tile = TMEM lanes
constexpr int kBN = 128;       // keys per tile
constexpr float kTau = 8.0f;   // lazy-rescale threshold (log2 units)
#ifndef FA_POLY_PAIRS
#define FA_POLY_PAIRS 0
#endif
// Of every 16 column pairs, this many use the FMA-pipe exp2 (the rest use MUFU).
constexpr int kPolyPairs = FA_POLY_PAIRS;
#ifndef FA_S_SPLIT
#define FA_S_SPLIT 1
#endif
// At D = 64: the keys 0-63 of S_{j+1} are computed once the first half of P_j
// is out (the softmax read all of S_j before writing it, and P_j only occupies
// columns 64-127), so only the other half of S_{j+1} remains between the
// release of P_j's second half and the next softmax (D = 64 is bound by that chain:
// 0.1219 vs 0.1259 ms on the (2, 8, 4096, 64) workload).  At D = 128 the two
// N = 64 products read Q from shared memory twice, and the S products are
// already at the shared-memory bandwidth limit: measured 8 % slower there.
template <int D>
constexpr bool split_s() { return FA_S_SPLIT != 0 && D == 64; }
#ifndef FA_MAX_CHAINS
#define FA_MAX_CHAINS 4
#endif
constexpr int kMaxChains = FA_MAX_CHAINS;   // independent chains of the row maximum
constexpr int kThreads = 384;
constexpr uint32_t kRegsControl = 72;    // warps 8-11
constexpr uint32_t kRegsSoftmax = 216;   // warps 0-7
static_assert(kRegsControl * 128 + kRegsSoftmax * 256 <= 384 * 168, "register split");

constexpr int kSchedMax = 2048;   // entries of the work-sorted list of ragged batches

// SCHED: the ragged and paged kernels keep their work-sorted (pair, sequence)
// list in shared memory.  The dense kernel instead stages its epilogue there:
// per softmax warp a 32-row x 64-column bf16/fp16 box of O (4 KB, laid out as
// the 128-byte swizzle of the O tensor map) and the warp's 32 LSE values, which
// the TMA engine writes to global memory.
template <int D, bool SCHED = false>
struct FwdLayout {
  static constexpr int kChunks = D / 64;              // 128-byte swizzle atoms along D
  static constexpr int kChunkBytes = kBM * 128;       // one atom column of a 128-row tile
  static constexpr int kTileBytes = kBM * D * 2;      // a 128-row tile of Q, K or V
  static constexpr int kSlots = D == 128 ? 4 : 8;     // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 4 + 2 + 1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem address, abort, list size, ok
  static constexpr int kSchedOff = kMiscOff + 16;
  static constexpr int kStageOBytes = 32 * 128;              // one warp's O box
  static constexpr int kStageOff = (kSchedOff + 1023) & ~1023;   // swizzle atoms: 1024-aligned
  static constexpr int kStageLseOff = kStageOff + 8 * kStageOBytes;
  static constexpr int kSmemBytes =
      (SCHED ? kSchedOff + kSchedMax * 4 : kStageLseOff + 8 * 32 * 4) +
      1024;                                                  // + slack for 1024-byte alignment
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct FwdParams {
  void* o;
  float* lse;
  // Ragged batch packed without padding (null: the dense [B, H, N, D] layout):
  // sequence b owns query rows [cu_q[b], cu_q[b+1]) of q/o [total_q, Hq, D] and
  // key rows [cu_k[b], cu_k[b+1]) of k/v [total_k, Hkv, D]; lse is [Hq, total_q].
  // Nq, Nk then bound the sequence lengths.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  // Paged keys/values (cu_k unused): sequence b's keys are the first seq_lens_k[b]
  // tokens of its pages block_table[b][0 ..] in the pool k/v [num_pages, 16, Hkv, D].
  const int* block_table;
  const int* seq_lens_k;
  int max_pages, num_pages;
  int B, Hq, Hkv, Nq, Nk;
  int num_mpairs;
  int num_items;      // num_mpairs * B * Hq work items, heaviest first
  int causal;
  int lse_bulk;       // dense: LSE rows leave by bulk copies (Nq % 4 == 0, lse 16-byte aligned)
  float scale_log2;   // scale * log2(e)
  int* err;
  uint64_t timeout_ns;
};

// Key tiles needed by the query tile starting at first_row of a sequence with Nq
// queries and Nk keys.
__device__ __forceinline__ int kv_tiles_for(int first_row, int Nq, int Nk, int causal) {
  if (first_row >= Nq) return 0;
  const int nk_tiles = (Nk + kBN - 1) / kBN;
  if (!causal) return nk_tiles;
  const int last_row = min(first_row + kBM - 1, Nq - 1);
  const int max_key = last_row + (Nk - Nq);
  return min(nk_tiles, max_key / kBN + 1);
}

// A work item: (sequence b, query head h, pair of 128-row query tiles).
struct FwdItem {
  int bh, b, h, hkv, q_row0, n0, n1;
  int q_start, k_start, nq, nk;   // the sequence's rows (dense: 0, 0, Nq, Nk)
};

// Batch layouts (kernel instantiations): dense [B, H, N, D]; ragged (packed
// [total, H, D] queries and keys with row offsets); paged (packed queries, keys
// and values in a page pool reached through a block table).
enum : int { kDense = 0, kRagged = 1, kPaged = 2 };
constexpr int kPageTok = 16;   // tokens per page of a paged pool

// Rows of sequence b of a ragged or paged batch, or false when its offsets or
// length break the rules (negative length, past the packed tensor or the block
// table, longer than the bound, causal with more queries than keys).
template <int MODE>
__device__ __forceinline__ bool ragged_rows(const FwdParams& p, int b, int& q0, int& nq, int& k0,
                                            int& nk) {
  q0 = __ldg(p.cu_q + b);
  const int q1 = __ldg(p.cu_q + b + 1);
  nq = q1 - q0;
  bool ok = q0 >= 0 && nq >= 0 && q1 <= p.total_q && nq <= p.Nq;
  if constexpr (MODE == kPaged) {
    k0 = 0;
    nk = __ldg(p.seq_lens_k + b);
    ok = ok && nk >= 0 && nk <= p.max_pages * kPageTok;
  } else {
    k0 = __ldg(p.cu_k + b);
    const int k1 = __ldg(p.cu_k + b + 1);
    nk = k1 - k0;
    ok = ok && k0 >= 0 && nk >= 0 && k1 <= p.total_k;
  }
  return ok && !(p.causal && nq > nk);
}
template <int MODE>
__device__ __forceinline__ int ragged_pairs(const FwdParams& p, int b) {
  int q0, nq, k0, nk;
  return ragged_rows<MODE>(p, b, q0, nq, k0, nk) ? (nq + 2 * kBM - 1) / (2 * kBM) : 0;
}

template <int MODE>
__device__ __forceinline__ FwdItem make_item(const FwdParams& p, int b, int h, int mpair) {
  FwdItem it;
  it.b = b;
  it.h = h;
  it.bh = b * p.Hq + h;
  it.hkv = h / (p.Hq / p.Hkv);
  it.q_row0 = mpair * 2 * kBM;
  if constexpr (MODE != kDense) {
    if (!ragged_rows<MODE>(p, b, it.q_start, it.nq, it.k_start, it.nk)) it.nq = it.nk = 0;
  } else {
    it.q_start = 0;
    it.k_start = 0;
    it.nq = p.Nq;
    it.nk = p.Nk;
  }
  it.n0 = kv_tiles_for(it.q_row0, it.nq, it.nk, p.causal);
  it.n1 = kv_tiles_for(it.q_row0 + kBM, it.nq, it.nk, p.causal);
  return it;
}

// The items of one CTA, in order.  The list is ordered by tile pair (heaviest
// first when causal), then sequence, then head; CTA c takes the r-th entry of
// rounds of gridDim entries, alternately left to right and right to left (with
// the heaviest-first order this balances the CTAs' totals about as well as
// handing items out dynamically).  Dense batches index the list in closed form.
// Ragged batches list only pairs that start inside their sequence (pair m of
// sequence b for m < ceil(Nq_b / 256)), so the rounds contain no empty items;
// every role of the CTA walks a cursor along that list, whose indices only grow.
// When the list is small enough (<= 2048 (pair, sequence) entries, B <= 1024,
// pairs <= 1024, <= 4095 key tiles) the CTA first sorts it by each entry's key
// tiles, heaviest first, in shared memory, so that the snake rounds balance
// sequences of very different lengths too.  (Separate instantiations keep the
// dense kernel free of all this.)
template <int MODE>
struct ItemWalker {
  int cta, C, r, total;
  int idx, m, b, h;   // ragged cursor: list entry idx is (pair m, sequence b, head h)
  const uint32_t* sorted;   // ragged: work-sorted (pair, sequence) keys, or null

  __device__ void init(const FwdParams& p, int cta_, int C_, const uint32_t* sorted_ = nullptr,
                       int n_sorted = 0) {
    cta = cta_;
    C = C_;
    r = 0;
    sorted = sorted_;
    if constexpr (MODE == kDense) {
      total = p.num_items;
      return;
    }
    if (sorted) {
      total = n_sorted * p.Hq;
      return;
    }
    int sum = 0, pmax = 0;
    for (int bb = 0; bb < p.B; ++bb) {
      const int pb = ragged_pairs<MODE>(p, bb);
      sum += pb;
      pmax = max(pmax, pb);
    }
    total = sum * p.Hq;
    idx = 0;
    h = 0;
    m = pmax - 1;
    b = 0;
    if (total > 0)
      while (ragged_pairs<MODE>(p, b) <= m) ++b;
  }
  // Moves the ragged cursor to list entry `target` (>= idx, < total).
  __device__ void advance(const FwdParams& p, int target) {
    int k = target - idx;
    while (k > 0) {
      const int left = p.Hq - h;
      if (k < left) {
        h += k;
        break;
      }
      k -= left;
      h = 0;
      do {
        ++b;
      } while (b < p.B && ragged_pairs<MODE>(p, b) <= m);
      if (b == p.B) {                            // next (lighter) pair of every sequence
        --m;
        b = 0;
        while (b < p.B && ragged_pairs<MODE>(p, b) <= m) ++b;
      }
    }
    idx = target;
  }
  __device__ bool next(const FwdParams& p, FwdItem& it) {
    const int i = r * C + ((r & 1) ? C - 1 - cta : cta);
    ++r;
    if (i >= total) return false;
    if constexpr (MODE != kDense) {
      if (sorted) {
        const int e = i / p.Hq;
        const uint32_t key = sorted[e];
        it = make_item<MODE>(p, static_cast<int>(key & 1023u),
                             i - e * p.Hq, 1023 - static_cast<int>((key >> 10) & 1023u));
        return true;
      }
      advance(p, i);
      it = make_item<MODE>(p, b, h, m);
    } else {
      const int BH = p.B * p.Hq;
      const int mrev = i / BH;
      const int bh = i - mrev * BH;
      const int b_ = bh / p.Hq;
      it = make_item<kDense>(p, b_, bh - b_ * p.Hq, p.causal ? (p.num_mpairs - 1 - mrev) : mrev);
    }
    return true;
  }
};

template <int D, bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  constexpr bool RAGGED = MODE != kDense;
  using L = FwdLayout<D, RAGGED>;
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
  auto kv_empty = [&](int s) { return bar(2 + L::kSlots + s); };
  auto s_full = [&](int t) { return bar(2 + 2 * L::kSlots + t); };
  // P is released in two halves (keys 0-63, 64-127) so that the first half of
  // P V runs while the second half of P is still being computed.
  auto p_half = [&](int t, int h) { return bar(4 + 2 * L::kSlots + 2 * t + h); };
  auto o_full = [&](int t) { return bar(8 + 2 * L::kSlots + t); };
  const uint32_t mma_done = bar(10 + 2 * L::kSlots);
  // Q smem may be refilled: every S MMA of the item has read it
  const uint32_t q_empty = bar(11 + 2 * L::kSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (RAGGED && cta == 0 && tid == 0) {
    for (int b = 0; b < p.B; ++b) {
      int q0, nq, k0, nk;
      if (!ragged_rows<MODE>(p, b, q0, nq, k0, nk)) {
        atomicOr(p.err, kErrBadIndex);           // that sequence is skipped
        break;
      }
    }
  }
  if (tid == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_half(t, 0), kBM);
      mbar_init(p_half(t, 1), kBM);
      mbar_init(o_full(t), 1);
    }
    for (int s = 0; s < L::kSlots; ++s) {
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
  // Ragged batches: the (pair, sequence) entries in shared memory, sorted by key
  // (4095 - key tiles) << 20 | (1023 - pair) << 10 | sequence, ascending.
  const uint32_t* sorted = nullptr;
  int n_sorted = 0;
  if constexpr (RAGGED) {
    uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::kSchedOff);
    int* list_n = reinterpret_cast<int*>(smem + L::kMiscOff + 8);
    volatile int* list_ok = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 12);
    if (tid == 0) {
      *list_n = 0;
      *list_ok = p.B <= 1024 ? 1 : 0;
    }
    __syncthreads();
    if (*list_ok) {
      for (int bb = tid; bb < p.B; bb += kThreads) {
        int q0, nq, k0, nk;
        if (!ragged_rows<MODE>(p, bb, q0, nq, k0, nk)) continue;
        const int pairs = (nq + 2 * kBM - 1) / (2 * kBM);
        for (int m = 0; m < pairs; ++m) {
          const int w = max(kv_tiles_for(m * 2 * kBM, nq, nk, p.causal),
                            kv_tiles_for(m * 2 * kBM + kBM, nq, nk, p.causal));
          const int at = atomicAdd(list_n, 1);
          if (at < kSchedMax && m < 1024 && w < 4096)
            list[at] = (static_cast<uint32_t>(4095 - w) << 20) |
                       (static_cast<uint32_t>(1023 - m) << 10) | static_cast<uint32_t>(bb);
          else
            *list_ok = 0;
        }
      }
    }
    __syncthreads();
    if (*list_ok) {
      // the keys are distinct, so the sorted order does not depend on the order
      // in which the threads appended them: bitonic sort, padded to a power of 2
      const int E = *list_n;
      int N = 1;
      while (N < E) N <<= 1;
      for (int i = E + tid; i < N; i += kThreads) list[i] = 0xffffffffu;
      __syncthreads();
      for (int k = 2; k <= N; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int i = tid; i < N; i += kThreads) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const uint32_t a = list[i], c2 = list[ixj];
              if ((a > c2) == ((i & k) == 0)) {
                list[i] = c2;
                list[ixj] = a;
              }
            }
          }
          __syncthreads();
        }
      }
      sorted = list;
      n_sorted = E;
    }
  }
  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == 8) {
      // ------------------------------------------------------------ TMA producer
      // Items in order; per item both Q tiles (a tile past Nq reads as zeros),
      // then K_j, V_j through the ring, whose position runs on across items.
      if constexpr (MODE == kPaged) {
        // A key tile is eight 16-token pages: the whole warp walks the items and
        // waits (warp-uniform), lane 0 posts each tile's bytes, and lane
        // pg * kChunks + ch reads page pg's block-table entry and issues its
        // chunk ch box, so the 8 (or 16) boxes and table reads leave together.
        // Keys past the sequence read its first page (masked later, but finite);
        // an id outside the pool is flagged and replaced by page 0.
        if (lane == 0) {
          tma_prefetch_desc(&tmQ);
          tma_prefetch_desc(&tmK);
          tma_prefetch_desc(&tmV);
        }
        auto wait_all = [&](uint32_t br, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait(br, parity, abort_flag, p.err, p.timeout_ns));
        };
        constexpr int kBoxes = (kBN / kPageTok) * L::kChunks;
        const int pg = lane / L::kChunks, ch = lane % L::kChunks;
        int pos = 0, items = 0;
        bool ok = true;
        ItemWalker<MODE> walk;
        walk.init(p, cta, C, sorted, n_sorted);
        FwdItem it;
        while (ok && walk.next(p, it)) {
          const int n_max = max(it.n0, it.n1);
          if (n_max == 0) continue;
          if (items > 0 && !wait_all(q_empty, (items - 1) & 1)) break;
          if (lane == 0) {
            for (int t = 0; t < 2; ++t) {
              mbar_arrive_expect_tx(q_full(t), L::kTileBytes);
              const uint32_t dst = sbase + L::kQOff + t * L::kTileBytes;
              for (int c2 = 0; c2 < L::kChunks; ++c2)   // [total_q, Hq, D]: box {64, 1, 128}
                tma_load_3d(dst + c2 * L::kChunkBytes, &tmQ, q_full(t), c2 * 64, it.h,
                            it.q_start + it.q_row0 + t * kBM);
            }
          }
          ++items;
          const int* tab = p.block_table + static_cast<size_t>(it.b) * p.max_pages;
          for (int j = 0; j < n_max && ok; ++j) {
            // this lane's page of key tile j, shared by its K and V boxes
            int page = 0;
            if (lane < kBoxes) {
              const int tok = j * kBN + pg * kPageTok;
              page = __ldg(tab + (tok < it.nk ? tok / kPageTok : 0));
              if (page < 0 || page >= p.num_pages) {
                atomicOr(p.err, kErrBadIndex);
                page = 0;
              }
            }
            for (int w = 0; w < 2; ++w, ++pos) {
              const int slot = pos % L::kSlots;
              const uint32_t ph = (pos / L::kSlots) & 1;
              if (!wait_all(kv_empty(slot), ph ^ 1)) {
                ok = false;
                break;
              }
              if (lane == 0) mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
              __syncwarp();
              const uint32_t dst = sbase + L::kKVOff + slot * L::kTileBytes;
              const void* tm = w ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmK);
              if (lane < kBoxes)
                tma_load_3d(dst + ch * L::kChunkBytes + pg * kPageTok * 128, tm, kv_full(slot),
                            ch * 64, it.hkv, page * kPageTok);
            }
          }
        }
        // Every issued copy must land before the CTA may exit (also on abort).
        if (lane == 0) {
          volatile int no_abort = 0;
          if (items > 0)
            for (int t = 0; t < 2; ++t)
              mbar_wait(q_full(t), (items - 1) & 1, &no_abort, p.err, p.timeout_ns);
          for (int sl = 0; sl < L::kSlots && sl < pos; ++sl) {
            const int last = sl + ((pos - 1 - sl) / L::kSlots) * L::kSlots;
            mbar_wait(kv_full(sl), (last / L::kSlots) & 1, &no_abort, p.err, p.timeout_ns);
          }
        }
      } else if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int pos = 0, items = 0;
        bool ok = true;
        ItemWalker<MODE> walk;
        walk.init(p, cta, C, sorted, n_sorted);
        FwdItem it;
        while (ok && walk.next(p, it)) {
          const int n_max = max(it.n0, it.n1);
          if (n_max == 0) continue;
          if (items > 0 && !mbar_wait(q_empty, (items - 1) & 1, abort_flag, p.err, p.timeout_ns))
            break;
          for (int t = 0; t < 2; ++t) {
            mbar_arrive_expect_tx(q_full(t), L::kTileBytes);
            const uint32_t dst = sbase + L::kQOff + t * L::kTileBytes;
            for (int ch = 0; ch < L::kChunks; ++ch) {
              if (RAGGED)   // [total_q, Hq, D]: box {64, 1 head, 128 rows}
                tma_load_3d(dst + ch * L::kChunkBytes, &tmQ, q_full(t), ch * 64, it.h,
                            it.q_start + it.q_row0 + t * kBM);
              else          // [B * Hq, Nq, D]: box {64, 128 rows, 1}
                tma_load_3d(dst + ch * L::kChunkBytes, &tmQ, q_full(t), ch * 64,
                            it.q_row0 + t * kBM, it.bh);
            }
          }
          ++items;
          const int kv_z = it.b * p.Hkv + it.hkv;
          for (int j = 0; j < n_max && ok; ++j) {
            for (int w = 0; w < 2; ++w, ++pos) {
              const int slot = pos % L::kSlots;
              const uint32_t ph = (pos / L::kSlots) & 1;
              if (!mbar_wait(kv_empty(slot), ph ^ 1, abort_flag, p.err, p.timeout_ns)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(kv_full(slot), L::kTileBytes);
              const uint32_t dst = sbase + L::kKVOff + slot * L::kTileBytes;
              const void* tm = w ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmK);
              for (int ch = 0; ch < L::kChunks; ++ch) {
                if (RAGGED)
                  tma_load_3d(dst + ch * L::kChunkBytes, tm, kv_full(slot), ch * 64, it.hkv,
                              it.k_start + j * kBN);
                else
                  tma_load_3d(dst + ch * L::kChunkBytes, tm, kv_full(slot), ch * 64,
                              j * kBN, kv_z);
              }
            }
          }
        }
        // Every issued copy must land before the CTA may exit (also on abort).
        volatile int no_abort = 0;
        if (items > 0)
          for (int t = 0; t < 2; ++t)
            mbar_wait(q_full(t), (items - 1) & 1, &no_abort, p.err, p.timeout_ns);
        for (int sl = 0; sl < L::kSlots && sl < pos; ++sl) {
          const int last = sl + ((pos - 1 - sl) / L::kSlots) * L::kSlots;
          mbar_wait(kv_full(sl), (last / L::kSlots) & 1, &no_abort, p.err, p.timeout_ns);
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      // The whole warp runs the waits, loop counters and descriptor arithmetic
      // (all warp-uniform); one elected lane issues the MMAs and commits.
      {
        const bool leader = elect_one();
        constexpr uint32_t idesc_s = idesc_f16(kBM, kBN, BF16, false);
        constexpr uint32_t idesc_pv = idesc_f16(kBM, D, BF16, true);
        auto slot_of = [&](int pos) { return pos % L::kSlots; };
        auto phase_of = [&](int pos) { return static_cast<uint32_t>((pos / L::kSlots) & 1); };
        auto wait = [&](uint32_t bar, uint32_t parity) {
          return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.err, p.timeout_ns));
        };
        auto commit = [&](uint32_t bar) {
          if (leader) tc_commit(bar);
        };
        // Descriptors are built once; moving to another K step or ring slot only
        // adds (byte offset >> 4) to the start-address field in the low bits.
        const uint64_t desc_q0 = smem_desc_sw128(sbase + L::kQOff, 16, 1024);
        const uint64_t desc_q1 = smem_desc_sw128(sbase + L::kQOff + L::kTileBytes, 16, 1024);
        const uint64_t desc_k = smem_desc_sw128(sbase + L::kKVOff, 16, 1024);            // K-major
        const uint64_t desc_v = smem_desc_sw128(sbase + L::kKVOff, L::kChunkBytes, 1024);  // MN-major
        // S_t = Q_t K^T : M=128, N=128, K=D in steps of 16 (32 bytes inside a swizzle atom)
        auto issue_s = [&](int t, int slot) {
          const uint64_t a0 = t ? desc_q1 : desc_q0;
          const uint64_t b0 = desc_k + static_cast<uint64_t>((slot * L::kTileBytes) >> 4);
          const uint32_t d = tmem + t * 128;
          if (leader) {
  #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off =
                  static_cast<uint64_t>(((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4);
              mma_ss(d, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
            }
            tc_commit(s_full(t));
          }
        };
        // Keys [key0, key0 + 64) of S_t = Q_t K^T into its columns key0 ..: the
        // K rows start key0 * 128 bytes into each swizzle-atom column (a whole
        // number of 8-row atoms); the second call commits S_t as complete.
        constexpr uint32_t idesc_s64 = idesc_f16(kBM, kBN / 2, BF16, false);
        auto issue_s_keys = [&](int t, int slot, int key0, bool last) {
          const uint64_t a0 = t ? desc_q1 : desc_q0;
          const uint64_t b0 =
              desc_k + static_cast<uint64_t>((slot * L::kTileBytes + key0 * 128) >> 4);
          const uint32_t d = tmem + t * 128 + key0;
          if (leader) {
  #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off =
                  static_cast<uint64_t>(((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4);
              mma_ss(d, a0 + off, b0 + off, idesc_s64, kk > 0 ? 1u : 0u);
            }
            if (last) tc_commit(s_full(t));
          }
        };
        // O_t += P_t V over keys [64 h, 64 h + 64): A = P from TMEM (bf16 pairs),
        // B = V tile, MN-major (D contiguous)
        auto issue_pv_half = [&](int t, int slot, int h, bool accumulate) {
          const uint64_t b0 = desc_v + static_cast<uint64_t>((slot * L::kTileBytes) >> 4);
          const uint32_t d = tmem + 256 + t * D;
          const uint32_t a = tmem + t * 128 + 64;   // P: 16-bit pairs in S's columns 64-127
          if (leader) {
  #pragma unroll
            for (int k4 = 0; k4 < kBN / 32; ++k4) {
              const int kk = h * (kBN / 32) + k4;
              mma_ts(d, a + kk * 8, b0 + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                     (accumulate || kk > 0) ? 1u : 0u);
            }
          }
        };
        bool ok = true;
        int pos = 0, items = 0;
        int tiles[2] = {0, 0};   // S tiles of each query-tile slot in earlier items (phases)
        ItemWalker<MODE> walk;
        walk.init(p, cta, C, sorted, n_sorted);
        FwdItem it;
        while (ok && walk.next(p, it)) {
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
            bool k_ready = false;   // K_{j+1} is waited for just before its first use
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int nt = t ? it.n1 : it.n0;
              if (!ok || j >= nt) continue;
              const uint32_t par = static_cast<uint32_t>((tiles[t] + j) & 1);
              ok = wait(p_half(t, 0), par);
              if (!ok) continue;
              tc_fence_after();
              issue_pv_half(t, slot_of(vpos), 0, j > 0);
              if constexpr (split_s<D>()) {
                // P_t(j)'s first half is out, so the softmax has read all of S_t(j):
                // keys 0-63 of S_t(j + 1) go into columns P_t(j) does not use
                if (j + 1 < nt) {
                  if (!k_ready) {
                    ok = wait(kv_full(slot_of(kpos)), phase_of(kpos));
                    k_ready = true;
                    if (!ok) continue;
                    tc_fence_after();
                  }
                  issue_s_keys(t, slot_of(kpos), 0, false);
                }
              }
              ok = wait(p_half(t, 1), par);
              if (!ok) continue;
              tc_fence_after();
              issue_pv_half(t, slot_of(vpos), 1, true);
              if (j + 1 < nt) {
                if constexpr (split_s<D>()) {
                  issue_s_keys(t, slot_of(kpos), kBN / 2, true);   // after P V has read P_t(j)
                } else {
                  if (!k_ready) {
                    ok = wait(kv_full(slot_of(kpos)), phase_of(kpos));
                    k_ready = true;
                    if (!ok) continue;
                    tc_fence_after();
                  }
                  issue_s(t, slot_of(kpos));
                }
              } else {
                commit(o_full(t));
              }
            }
            if (!ok) break;
            if (j + 2 == n_max) commit(q_empty);   // the item's last S MMAs are issued
            commit(kv_empty(slot_of(vpos)));
            if (has_next) commit(kv_empty(slot_of(kpos)));
          }
          pos += 2 * n_max;
          tiles[0] += it.n0;
          tiles[1] += it.n1;
        }
        // All issued MMAs must complete before TMEM is released (also on abort).
        commit(mma_done);
        volatile int no_abort = 0;
        mbar_wait(mma_done, 0, &no_abort, p.err, p.timeout_ns);
      }
    }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tP = tS + 64;             // P as 16-bit pairs over S's keys 64-127
    const uint32_t tO = tmem + lane_base + 256 + t * D;
    int tiles = 0, outs = 0;     // S tiles and O tiles of this slot in earlier items (phases)
    bool ok = true;
    ItemWalker<MODE> walk;
    walk.init(p, cta, C, sorted, n_sorted);
    FwdItem it;
    while (ok && walk.next(p, it)) {
    const int q_row0 = it.q_row0;
    const int row = q_row0 + t * kBM + r;          // within the sequence
    const int n = t ? it.n1 : it.n0;
    // o element offset / D and lse offset of this row
    const size_t o_index = RAGGED
        ? static_cast<size_t>(it.q_start + row) * p.Hq + it.h
        : static_cast<size_t>(it.bh) * p.Nq + row;
    const size_t row_index = RAGGED
        ? static_cast<size_t>(it.h) * p.total_q + it.q_start + row
        : o_index;
    using Out = uint16_t;
    Out* o_row = reinterpret_cast<Out*>(p.o) + o_index * D;
    if (n == 0) {
      if (max(it.n0, it.n1) == 0 && row < it.nq) {   // only reached when Nk == 0
        uint4 z = make_uint4(0, 0, 0, 0);
        for (int ch = 0; ch < D / 8; ++ch) reinterpret_cast<uint4*>(o_row)[ch] = z;
        if (p.lse) p.lse[row_index] = -INFINITY;
      }
    } else {
      float m_used = -INFINITY;
      float l = 0.f;
      const int off = it.nk - it.nq;
      const int tile_first = q_row0 + t * kBM;
      for (int j = 0; j < n; ++j) {
        // tcgen05.ld/st/wait are warp-collective: every branch around them is
        // made warp-uniform, also on the abort path.
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
            (kbase + kBN > it.nk) || (p.causal && kbase + kBN - 1 > tile_first + off);
        if (need_mask) {
          int lim = it.nk - 1 - kbase;                      // last visible column
          if (p.causal) lim = min(lim, row + off - kbase);
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > lim) s[e] = __float_as_uint(-INFINITY);
        }
        const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
        uint64_t sum2[4] = {0, 0, 0, 0};   // four independent packed partial sums
        // exponentials of the 32 columns 32 c .. 32 c + 31 against reference -nm,
        // packed to 16-bit pairs (unmasked tiles may put the first kPolyPairs
        // pairs of every 32 columns on the FMA pipe)
        auto exp_cols = [&](int c, float nm, uint32_t (&pk)[16]) {
          const uint64_t nm2 = f2_pack(nm, nm);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1, p0, p1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[32 * c + 2 * e]),
                                     __uint_as_float(s[32 * c + 2 * e + 1])), c2, nm2), x0, x1);
            if (!need_mask && e < kPolyPairs) {
              exp2_fma_pair(x0, x1, p0, p1);
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            sum2[e & 3] = f2_add(sum2[e & 3], f2_pack(p0, p1));
            pk[e] = BF16 ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
          }
        };
        // row maximum: kMaxChains independent three-input-max chains, then a short tree
        float acc[kMaxChains];
#pragma unroll
        for (int k = 0; k < kMaxChains; ++k) acc[k] = __uint_as_float(s[k]);
#pragma unroll
        for (int e = kMaxChains; e + 2 * kMaxChains <= 128; e += 2 * kMaxChains)
#pragma unroll
          for (int k = 0; k < kMaxChains; ++k)
            acc[k] = fmax3(acc[k], __uint_as_float(s[e + k]),
                           __uint_as_float(s[e + kMaxChains + k]));
#pragma unroll
        for (int k = 0; k < kMaxChains; ++k)
          acc[k] = fmaxf(acc[k], __uint_as_float(s[128 - kMaxChains + k]));
#pragma unroll
        for (int k = 1; k < kMaxChains; ++k) acc[0] = fmaxf(acc[0], acc[k]);
        const float mx = acc[0];
        const float m_tile = mx * p.scale_log2;
        const bool move = m_tile > m_used + kTau;
        float alpha = 1.f;
        if (move) {
          alpha = ex2(m_used - m_tile);   // 0 on the first visible tile
          l *= alpha;
          m_used = m_tile;
        }
        // Rescale O rows whose reference moved; the whole warp takes part in
        // the TMEM round trip, rows that did not move keep alpha = 1.
        if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov, p.err);
            tmem_wait_ld(p.err);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + 32 * c, ov, p.err);
          }
        }
        const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
          exp_cols(c, neg_m, pk);
          tmem_st16(tP + 16 * c, pk, p.err);
        }
        tmem_wait_st(p.err);                 // keys 0-63 of P are in place
        tc_fence_before();
        mbar_arrive(p_half(t, 0));
#pragma unroll
        for (int c = 2; c < 4; ++c) {
          uint32_t pk[16];
          exp_cols(c, neg_m, pk);
          tmem_st16(tP + 16 * c, pk, p.err);
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
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float lse_v =
            l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        if constexpr (MODE == kDense) {
          // TMA epilogue.  Per 64-column half, the warp's 32 rows go to its
          // staging box (128-byte swizzle: 16-byte chunk k of row r at k ^ (r & 7),
          // conflict-free), then one lane stores the box through the O tensor map,
          // which clips rows past Nq; the LSE values leave by one bulk copy.
          const uint32_t stage = sbase + L::kStageOff + warp * L::kStageOBytes;
          const int row0 = tile_first + (warp & 3) * 32;   // the warp's first row
          const bool slab_live = row0 < it.nq;              // warp-uniform
#pragma unroll 1
          for (int hh = 0; hh < D / 64; ++hh) {
            if (lane == 0) bulk_wait_read_all();   // earlier boxes have left the stage
            __syncwarp();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              uint32_t ov[32];
              tmem_ld32(tO + 64 * hh + 32 * cc, ov, p.err);
              tmem_wait_ld(p.err);
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float a = __uint_as_float(ov[2 * e]) * inv_l;
                const float bb = __uint_as_float(ov[2 * e + 1]) * inv_l;
                pk[e] = BF16 ? pack_bf16x2(a, bb) : pack_f16x2(a, bb);
              }
#pragma unroll
              for (int v = 0; v < 4; ++v)
                st_shared_v4(stage + lane * 128 + (((cc * 4 + v) ^ (lane & 7)) << 4), pk[4 * v],
                             pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && slab_live) {
              tma_store_3d(&tmO, stage, 64 * hh, row0, it.bh);
              bulk_commit();
            }
          }
          if (p.lse) {
            if (p.lse_bulk) {
              const uint32_t lst = sbase + L::kStageLseOff + warp * 128;
              st_shared_f32(lst + lane * 4, lse_v);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0 && slab_live) {
                const int nrows = min(32, it.nq - row0);   // a multiple of 4 (Nq % 4 == 0)
                bulk_store(p.lse + static_cast<size_t>(it.bh) * p.Nq + row0, lst, nrows * 4);
                bulk_commit();
              }
            } else if (row < it.nq) {
              p.lse[row_index] = lse_v;
            }
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov, p.err);
            tmem_wait_ld(p.err);
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float a = __uint_as_float(ov[2 * e]) * inv_l;
              const float bb = __uint_as_float(ov[2 * e + 1]) * inv_l;
              pk[e] = BF16 ? pack_bf16x2(a, bb) : pack_f16x2(a, bb);
            }
            if (row < it.nq) {
              uint4* dst = reinterpret_cast<uint4*>(o_row + 32 * c);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
          if (p.lse && row < it.nq) p.lse[row_index] = lse_v;
        }
      }
    }
    }
    // the stores of the last epilogue complete before the CTA's shared memory goes
    if constexpr (MODE == kDense) {
      if (lane == 0) bulk_wait_all();
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

// ---------------------------------------------------------------- host side
// 3-D map over a contiguous [Z, N, D] tensor of 16-bit elements with a
// 64 x 128 x 1 box and 128-byte swizzle (one swizzle atom column per box).
int encode_3d(CUtensorMap* m, const void* base, bool bf16, int D, int N, int Z) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(Z)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                               static_cast<uint64_t>(N) * static_cast<uint64_t>(D) * 2};
  const uint32_t box[3] = {64, 128, 1};
  return encode_tensor_map_16bit(m, base, bf16, 3, dims, strides, box);
}
// Store map of the dense output O [Z, N, D]: a 64 x 32 x 1 box (one softmax
// warp's rows, one swizzle atom column) with 128-byte swizzle.
int encode_o_store(CUtensorMap* m, void* base, bool bf16, int D, int N, int Z) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(Z)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                               static_cast<uint64_t>(N) * static_cast<uint64_t>(D) * 2};
  const uint32_t box[3] = {64, 32, 1};
  return encode_tensor_map_16bit(m, base, bf16, 3, dims, strides, box);
}
// 3-D map over a packed [T, H, D] tensor (token-major) with a 64 x 1 x rows box:
// rows = 128 lands like encode_3d's box (128 rows of 128 bytes); rows = 16 is one
// page of a paged pool, eight of which fill the same tile.
int encode_packed(CUtensorMap* m, const void* base, bool bf16, int D, int H, int T,
                  int rows = 128) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(T)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                               static_cast<uint64_t>(H) * static_cast<uint64_t>(D) * 2};
  const uint32_t box[3] = {64, 1, static_cast<uint32_t>(rows)};
  return encode_tensor_map_16bit(m, base, bf16, 3, dims, strides, box);
}

int fwd_sm_count(int device) {
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

template <int D, bool BF16>
int launch_typed(const void* q, const void* k, const void* v, void* o, float* lse,
                 const FwdLayoutArgs& la, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                 int causal, cudaStream_t stream, int device) {
  const int* cu_q = la.cu_q;
  const int total_q = la.total_q, total_k = la.total_k;
  const bool paged = la.block_table != nullptr;
  using L = FwdLayout<D, false>;
  using LR = FwdLayout<D, true>;   // ragged and paged batches
  static int attr_gen[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> g(mu);
    if (device < 0 || device >= 64) return set_error(FA_ERR_CUDA, "device ordinal out of range");
    if (attr_gen[device] != cache_generation()) {
      cudaError_t e = cudaFuncSetAttribute(fa_fwd_kernel<D, BF16, kDense>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           L::kSmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fa_fwd_kernel<D, BF16, kRagged>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, LR::kSmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fa_fwd_kernel<D, BF16, kPaged>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, LR::kSmemBytes);
      if (e != cudaSuccess)
        return set_error(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      attr_gen[device] = cache_generation();
    }
  }
  CUtensorMap tq, tk, tv;
  int rc;
  if (cu_q) {
    if ((rc = encode_packed(&tq, q, BF16, D, Hq, total_q)) != FA_OK) return rc;
  } else if ((rc = encode_3d(&tq, q, BF16, D, Nq, B * Hq)) != FA_OK) {
    return rc;
  }
  if (paged) {
    const int pool_tok = la.num_pages * kPageTok;
    if ((rc = encode_packed(&tk, k, BF16, D, Hkv, pool_tok, kPageTok)) != FA_OK) return rc;
    if ((rc = encode_packed(&tv, v, BF16, D, Hkv, pool_tok, kPageTok)) != FA_OK) return rc;
  } else if (cu_q && total_k > 0) {
    if ((rc = encode_packed(&tk, k, BF16, D, Hkv, total_k)) != FA_OK) return rc;
    if ((rc = encode_packed(&tv, v, BF16, D, Hkv, total_k)) != FA_OK) return rc;
  } else if (!cu_q && Nk > 0) {
    if ((rc = encode_3d(&tk, k, BF16, D, Nk, B * Hkv)) != FA_OK) return rc;
    if ((rc = encode_3d(&tv, v, BF16, D, Nk, B * Hkv)) != FA_OK) return rc;
  } else {
    tk = tq;   // no key tile exists, so these maps are never read
    tv = tq;
  }
  CUtensorMap to = tq;   // ragged and paged batches store O with plain stores
  if (!cu_q && (rc = encode_o_store(&to, o, BF16, D, Nq, B * Hq)) != FA_OK) return rc;
  FwdParams prm;
  prm.o = o;
  prm.lse = lse;
  prm.lse_bulk = lse != nullptr && (Nq % 4) == 0 && (reinterpret_cast<uintptr_t>(lse) & 15u) == 0;
  prm.cu_q = cu_q;
  prm.cu_k = la.cu_k;
  prm.total_q = total_q;
  prm.total_k = total_k;
  prm.block_table = la.block_table;
  prm.seq_lens_k = la.seq_lens_k;
  prm.max_pages = la.max_pages;
  prm.num_pages = la.num_pages;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.num_mpairs = (Nq + 2 * kBM - 1) / (2 * kBM);
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.err = device_error_word(device);
  prm.timeout_ns = kWaitLimitNs;
  if (!prm.err) return set_error(FA_ERR_CUDA, "device error word unavailable");
  const long long items = static_cast<long long>(prm.num_mpairs) * B * Hq;
  if (items > 0x7fffffffLL) return set_error(FA_ERR_UNSUPPORTED, "too many work items");
  prm.num_items = static_cast<int>(items);
  // persistent: one CTA per SM (at most one per item), each walking its items
  const int nsm = fwd_sm_count(device);
  if (nsm <= 0) return set_error(FA_ERR_CUDA, "cannot read the SM count of device %d", device);
  const int grid = static_cast<int>(std::min<long long>(items, nsm));
  if (grid == 0) return FA_OK;
  const unsigned g = static_cast<unsigned>(grid);
  if (paged)
    fa_fwd_kernel<D, BF16, kPaged><<<g, kThreads, LR::kSmemBytes, stream>>>(tq, tk, tv, to, prm);
  else if (cu_q)
    fa_fwd_kernel<D, BF16, kRagged><<<g, kThreads, LR::kSmemBytes, stream>>>(tq, tk, tv, to, prm);
  else
    fa_fwd_kernel<D, BF16, kDense><<<g, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, to, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(FA_ERR_CUDA, "fa_fwd launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

}  // namespace

int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
               const FwdLayoutArgs& la, int B, int Hq, int Hkv, int Nq, int Nk, int D,
               float scale, int causal, bool bf16, cudaStream_t stream, int device) {
#define FA_FWD_ARGS q, k, v, o, lse, la, B, Hq, Hkv, Nq, Nk, scale, causal, stream, device
  if (D == 128)
    return bf16 ? launch_typed<128, true>(FA_FWD_ARGS) : launch_typed<128, false>(FA_FWD_ARGS);
  if (D == 64)
    return bf16 ? launch_typed<64, true>(FA_FWD_ARGS) : launch_typed<64, false>(FA_FWD_ARGS);
#undef FA_FWD_ARGS
  return set_error(FA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
}

}  // namespace fa
