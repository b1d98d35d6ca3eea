// Attention plan for the tensor-core attention path: targets in tiles of
// kTileM consecutive atoms of the traversal order, and per tile the sorted
// union of their neighbour lists with a (target x union) membership bitmask.
//
// The streaming attention of "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构"
// §3.2 processes each target independently; grouping spatially adjacent
// targets (the cell order of the graph builder) lets one tile read each
// neighbour row once for all of its targets, and the membership mask keeps
// the softmax exactly over each target's own neighbour list.
//
// One 256-thread CTA per tile builds the union from a shared-memory bitmap
// over atom indices (ascending atom index: a deterministic order) and sets one
// mask bit per (target, neighbour) at the position given by the bitmap's
// prefix counts.  The same CTA then writes the tile's target record: target
// ids, |r|^l and the real Wigner-D matrices of the targets' alignment
// rotations ([EX] §2.1), which the target coupling of the attention epilogue
// applies (one thread per target slot, after the union and mask; at lmax 3 a
// separate kernel writes the slots).
#include <type_traits>

#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kPlanThreads = 256;

struct PlanParams {
  const float* pos;      // [n][3] (the tile records' rotations)
  const int32_t* nbr;    // [n][K]
  const int32_t* cnt;    // [n] or null (then every slot is scanned, -1 skipped)
  const int32_t* order;  // [n] or null
  PlanView plan;
  int n, K;
};

// The record entries of target slot r of a tile: the slot's atom (-1 for an
// empty slot), |r|^l and the Wigner-D matrices of its alignment rotation
// (identity for an empty slot or an atom at the origin), built in registers.
// The header (union length, three zeros) is written by the caller.
template <int L>
__device__ __forceinline__ void write_slot_record(int tg, const float* __restrict__ pos, int r,
                                                  float* __restrict__ R) {
  constexpr int WS = wig_size(L);
  static_assert(WS == rec_wig_size(L) && plan_record_words(L) % 4 == 0, "record layout");
  float Q[9];
  float rr = 0.f;
  if (tg >= 0) rr = alignment_rotation(pos[3 * tg], pos[3 * tg + 1], pos[3 * tg + 2], Q);
  else alignment_rotation(0.f, 0.f, 0.f, Q);
  float D[WS];
  wigner_regs<L>(Q, D);
#pragma unroll
  for (int e = 0; e < WS; ++e) R[rec_off_D(L) + r * WS + e] = D[e];
  reinterpret_cast<int*>(R)[kRecTgt + r] = tg;
  float a = 1.f;
#pragma unroll
  for (int l = 0; l <= L; ++l) {
    R[kRecRp + r * (L + 1) + l] = a;
    a *= rr;
  }
}

// One CTA per tile.  Shared memory holds a bitmap over all atom indices
// (bit j set when atom j is a neighbour of some target of the tile), the
// per-word prefix counts of that bitmap, the tile's membership mask and its
// neighbour-list entries.
//  1. load the tile's entries (a thread's entries of all 16 rows in flight
//     together), keep them in shared memory and set the bit of every one;
//  2. prefix-count the bitmap's words: the union, in ascending atom index, is
//     read straight off the bitmap, and the union position of atom j is
//     prefix[j / 32] + popcount(bits of word j / 32 below j);
//  3. one membership bit per (target, neighbour) at that position.
// Cost per tile is O(n / 32) words plus O(16 K) entries; deterministic.
template <int L, bool RECORDS>
__global__ void __launch_bounds__(kPlanThreads, 6) build_plan_kernel(const __grid_constant__ PlanParams p) {
  extern __shared__ uint32_t sm[];
  const PlanView& pv = p.plan;
  const int cap = pv.cap;                         // >= kTileM * K, power of two
  const int words = cap / 32;                     // mask words per target row
  const int nw = (p.n + 31) / 32;                 // bitmap words
  uint32_t* bitmap = sm;                          // [nw]
  uint32_t* prefix = sm + nw;                     // [nw]
  uint32_t* mask = sm + 2 * nw;                   // [kTileM][words]
  int* ent = reinterpret_cast<int*>(mask + kTileM * words);   // [kTileM][K] the tile's entries
  __shared__ int tgt[kTileM], rowcnt[kTileM];
  __shared__ int warp_sum[kPlanThreads / 32];
  __shared__ int s_unique;
  if (blockIdx.x == 0 && threadIdx.x == 0) *pv.sched = 0;   // the attention kernel's claim counter
  const int tile = blockIdx.x;

  // the tile's targets and their neighbour counts (0 for an empty slot)
  if (threadIdx.x < kTileM) {
    const long long slot = (long long)tile * kTileM + threadIdx.x;
    int t = -1;
    if (slot < p.n) t = p.order ? p.order[slot] : int(slot);
    if ((unsigned)t >= (unsigned)p.n) t = -1;
    int c = 0;
    if (t >= 0) {
      c = p.cnt ? p.cnt[t] : p.K;
      c = c < 0 ? 0 : (c > p.K ? p.K : c);
    }
    tgt[threadIdx.x] = t;
    rowcnt[threadIdx.x] = c;
  }
  for (int i = threadIdx.x; i < nw; i += blockDim.x) bitmap[i] = 0u;
  for (int i = threadIdx.x; i < kTileM * words; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  // 1. the tile's entries and the bitmap of their union: thread t takes
  // entry e = t, t + 256, ... of every row (coalesced loads of nbr, eight
  // rows' loads in flight together); slots past a row's count hold -1
  constexpr int kBatch = 8;
  for (int e = threadIdx.x; e < p.K; e += blockDim.x) {
#pragma unroll 1
    for (int r0 = 0; r0 < kTileM; r0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        v[i] = e < rowcnt[r0 + i] ? p.nbr[(long long)tgt[r0 + i] * p.K + e] : -1;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        ent[(r0 + i) * p.K + e] = v[i];
        if ((unsigned)v[i] < (unsigned)p.n) atomicOr(&bitmap[v[i] >> 5], 1u << (v[i] & 31));
      }
    }
  }
  __syncthreads();
  // 2. per-word exclusive prefix counts (contiguous chunk per thread + block scan)
  const int per = (nw + kPlanThreads - 1) / kPlanThreads;
  const int w0 = threadIdx.x * per;
  const int w1 = min(w0 + per, nw);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bitmap[w]);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[wid] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) {
      const int v = warp_sum[w];
      warp_sum[w] = acc;
      acc += v;
    }
    s_unique = acc;
  }
  __syncthreads();
  const int U = s_unique;
  int* uni = pv.uni + (long long)tile * cap;
  {
    int pos = warp_sum[wid] + incl - mine;
    for (int w = w0; w < w1; ++w) {
      prefix[w] = uint32_t(pos);
      uint32_t b = bitmap[w];
      while (b) {
        const int bit = __ffs(b) - 1;
        uni[pos++] = w * 32 + bit;
        b &= b - 1;
      }
    }
  }
  __syncthreads();
  // pad the union to whole chunks of kPlanPad (at least one) with a valid
  // index whose mask bits stay zero
  const int upad = U > 0 ? (U + kPlanPad - 1) / kPlanPad * kPlanPad : kPlanPad;
  const int filler = U > 0 ? uni[0] : 0;
  for (int e = U + threadIdx.x; e < upad; e += blockDim.x) uni[e] = filler;
  if (threadIdx.x == 0) pv.ulen[tile] = U;
  // 3. membership bits, from the cached entries
  for (int r = 0; r < kTileM; ++r) {
    const int c = rowcnt[r];
    for (int e = threadIdx.x; e < c; e += blockDim.x) {
      const int j = ent[r * p.K + e];
      if ((unsigned)j >= (unsigned)p.n) continue;
      const int pos = int(prefix[j >> 5]) + __popc(bitmap[j >> 5] & ((1u << (j & 31)) - 1u));
      atomicOr(&mask[r * words + (pos >> 5)], 1u << (pos & 31));
    }
  }
  __syncthreads();
  // word-major in memory: the kTileM words of one 32-atom chunk are contiguous
  uint32_t* gmask = pv.mask + (long long)tile * words * kTileM;
  const int uw = upad / 32;
  for (int i = threadIdx.x; i < kTileM * uw; i += blockDim.x) {
    const int w = i / kTileM, r = i % kTileM;
    gmask[i] = mask[r * words + w];
  }
  // 4. the tile record: header, then one slot per thread of the first 16
  // (RECORDS; at lmax 3 the record's registers would cost the CTA its
  // occupancy, and tile_records_kernel writes the slots instead)
  float* R = pv.rec + (long long)tile * plan_record_words(L);
  if (threadIdx.x < kRecHdr) reinterpret_cast<int*>(R)[threadIdx.x] = threadIdx.x == 0 ? U : 0;
  if constexpr (RECORDS)
    if (threadIdx.x < kTileM) write_slot_record<L>(tgt[threadIdx.x], p.pos, threadIdx.x, R);
}

// The same plan for large n, at a cost per tile independent of n: one CTA per
// tile keeps a hash set of the tile's neighbour indices in shared memory
// (open addressing, 2 * cap slots, so it never fills), collects the distinct
// indices as they are inserted, sorts them by a block-wide bitonic sort, and
// sets each (target, neighbour) membership bit at the position a binary
// search of the sorted union gives.  Union, padding and mask are bit for bit
// those of build_plan_kernel.
template <int L, bool RECORDS>
__global__ void __launch_bounds__(kPlanThreads) build_plan_hash_kernel(const __grid_constant__ PlanParams p) {
  extern __shared__ int hsm[];
  const PlanView& pv = p.plan;
  const int cap = pv.cap;                         // >= kTileM * K, power of two
  const int words = cap / 32;
  const int hs = 2 * cap;                         // hash slots
  int* table = hsm;                               // [hs], -1 = empty
  int* srt = hsm + hs;                            // [cap] distinct indices, then sorted
  uint32_t* mask = reinterpret_cast<uint32_t*>(srt + cap);   // [kTileM][words]
  __shared__ int tgt[kTileM], rowcnt[kTileM];
  __shared__ int s_unique;
  if (blockIdx.x == 0 && threadIdx.x == 0) *pv.sched = 0;   // the attention kernel's claim counter
  const int tile = blockIdx.x;
  if (threadIdx.x < kTileM) {
    const long long slot = (long long)tile * kTileM + threadIdx.x;
    int t = -1;
    if (slot < p.n) t = p.order ? p.order[slot] : int(slot);
    if ((unsigned)t >= (unsigned)p.n) t = -1;
    int c = 0;
    if (t >= 0) {
      c = p.cnt ? p.cnt[t] : p.K;
      c = c < 0 ? 0 : (c > p.K ? p.K : c);
    }
    tgt[threadIdx.x] = t;
    rowcnt[threadIdx.x] = c;
  }
  if (threadIdx.x == 0) s_unique = 0;
  for (int i = threadIdx.x; i < hs; i += blockDim.x) table[i] = -1;
  for (int i = threadIdx.x; i < kTileM * words; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  auto for_each_entry = [&](auto&& f) {
    for (int r = 0; r < kTileM; ++r) {
      const int c = rowcnt[r];
      const int32_t* row = p.nbr + (long long)(tgt[r] < 0 ? 0 : tgt[r]) * p.K;
      for (int e = threadIdx.x; e < c; e += blockDim.x) f(r, row[e]);
    }
  };
  // 1. distinct indices (at most kTileM * K <= cap of them; the table has
  //    twice that many slots, so every probe sequence ends within hs steps)
  for_each_entry([&](int, int j) {
    if ((unsigned)j >= (unsigned)p.n) return;
    unsigned slot = (unsigned(j) * 2654435761u) & unsigned(hs - 1);
    for (int probe = 0; probe < hs; ++probe) {
      const int prev = atomicCAS(&table[slot], -1, j);
      if (prev == -1) {
        srt[atomicAdd(&s_unique, 1)] = j;
        return;
      }
      if (prev == j) return;
      slot = (slot + 1) & unsigned(hs - 1);
    }
  });
  __syncthreads();
  const int U = s_unique;
  // 2. bitonic sort of srt[0, P2), the tail filled with INT_MAX
  int P2 = 1;
  while (P2 < U) P2 <<= 1;
  for (int i = U + threadIdx.x; i < P2; i += blockDim.x) srt[i] = 0x7fffffff;
  __syncthreads();
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const int a = srt[i], b = srt[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            srt[i] = b;
            srt[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // 3. the union (ascending), padded as build_plan_kernel pads it
  int* uni = pv.uni + (long long)tile * cap;
  for (int i = threadIdx.x; i < U; i += blockDim.x) uni[i] = srt[i];
  const int upad = U > 0 ? (U + kPlanPad - 1) / kPlanPad * kPlanPad : kPlanPad;
  const int filler = U > 0 ? srt[0] : 0;
  for (int e = U + threadIdx.x; e < upad; e += blockDim.x) uni[e] = filler;
  if (threadIdx.x == 0) pv.ulen[tile] = U;
  // 4. membership bits at each neighbour's union position
  for_each_entry([&](int r, int j) {
    if ((unsigned)j >= (unsigned)p.n) return;
    int lo = 0, hi = U;                           // first position with srt >= j
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (srt[mid] < j) lo = mid + 1;
      else hi = mid;
    }
    atomicOr(&mask[r * words + (lo >> 5)], 1u << (lo & 31));
  });
  __syncthreads();
  uint32_t* gmask = pv.mask + (long long)tile * words * kTileM;
  const int uw = upad / 32;
  for (int i = threadIdx.x; i < kTileM * uw; i += blockDim.x) {
    const int w = i / kTileM, r = i % kTileM;
    gmask[i] = mask[r * words + w];
  }
  // 4. the tile record: header, then one slot per thread of the first 16
  // (RECORDS; at lmax 3 the record's registers would cost the CTA its
  // occupancy, and tile_records_kernel writes the slots instead)
  float* R = pv.rec + (long long)tile * plan_record_words(L);
  if (threadIdx.x < kRecHdr) reinterpret_cast<int*>(R)[threadIdx.x] = threadIdx.x == 0 ? U : 0;
  if constexpr (RECORDS)
    if (threadIdx.x < kTileM) write_slot_record<L>(tgt[threadIdx.x], p.pos, threadIdx.x, R);
}

// The record slots of every tile, one thread per slot (tile * kTileM + r),
// for plans whose builder does not write them (lmax 3).
constexpr int kRecThreads = 128;
template <int L>
__global__ void __launch_bounds__(kRecThreads)
tile_records_kernel(const int32_t* __restrict__ order, const float* __restrict__ pos, int n, int tiles,
                    float* __restrict__ rec) {
  const long long slot = (long long)blockIdx.x * kRecThreads + threadIdx.x;
  if (slot >= (long long)tiles * kTileM) return;
  int tg = -1;
  if (slot < n) tg = order ? order[slot] : int(slot);
  if ((unsigned)tg >= (unsigned)n) tg = -1;
  write_slot_record<L>(tg, pos, int(slot % kTileM), rec + (slot / kTileM) * plan_record_words(L));
}

}  // namespace

// Systems up to this many atoms use the bitmap builder (its two bitmaps take
// n / 4 bytes of shared memory and O(n / 32) work per tile); larger ones the
// hash builder, whose shared memory and work per tile depend only on K.
constexpr int kBitmapPlanAtoms = 1 << 17;

size_t plan_smem_bytes(int n, int K) {
  const size_t mask = size_t(kTileM) * (plan_capacity(K) / 32) * sizeof(uint32_t);
  if (n <= kBitmapPlanAtoms) {
    const size_t nw = (size_t(n) + 31) / 32;
    return 2 * nw * sizeof(uint32_t) + mask + size_t(kTileM) * K * sizeof(int);   // + entries
  }
  return size_t(3) * plan_capacity(K) * sizeof(int) + mask;   // table, sorted union, mask
}

int plan_capacity(int K) {
  int cap = 32;
  while (cap < kTileM * K) cap <<= 1;
  return cap;
}

size_t plan_bytes(int n, int K, int lmax) {
  const size_t tiles = (size_t(n) + kTileM - 1) / kTileM;
  const size_t cap = size_t(plan_capacity(K));
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  return a256(tiles * sizeof(int)) + a256(tiles * cap * sizeof(int)) +
         a256(tiles * kTileM * (cap / 32) * sizeof(uint32_t)) +
         a256(tiles * size_t(plan_record_words(lmax)) * sizeof(float)) + a256(sizeof(int));
}

PlanView plan_view(void* base, int n, int K, int lmax) {
  const size_t tiles = (size_t(n) + kTileM - 1) / kTileM;
  const int cap = plan_capacity(K);
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  PlanView v;
  char* b = static_cast<char*>(base);
  v.ulen = reinterpret_cast<int*>(b);
  b += a256(tiles * sizeof(int));
  v.uni = reinterpret_cast<int*>(b);
  b += a256(tiles * size_t(cap) * sizeof(int));
  v.mask = reinterpret_cast<uint32_t*>(b);
  b += a256(tiles * kTileM * (size_t(cap) / 32) * sizeof(uint32_t));
  v.rec = reinterpret_cast<float*>(b);
  b += a256(tiles * size_t(plan_record_words(lmax)) * sizeof(float));
  v.sched = reinterpret_cast<int*>(b);
  v.cap = cap;
  v.tiles = int(tiles);
  return v;
}

int launch_build_plan(int n, int K, int lmax, const int32_t* d_nbr, const int32_t* d_cnt,
                      const int32_t* d_order, const float* d_pos, void* d_plan, cudaStream_t st) {
  PlanParams p;
  p.nbr = d_nbr;
  p.cnt = d_cnt;
  p.order = d_order;
  p.plan = plan_view(d_plan, n, K, lmax);
  p.n = n;
  p.K = K;
  p.pos = d_pos;
  const size_t shmem = plan_smem_bytes(n, K);
  if (shmem > kPlanSmemLimit) return EGAT_ERR_UNSUPPORTED;
  auto pick = [&](auto lc) {
    constexpr int L = decltype(lc)::value;
    return n <= kBitmapPlanAtoms ? build_plan_kernel<L, (L < 3)> : build_plan_hash_kernel<L, (L < 3)>;
  };
  void (*kern)(PlanParams) = nullptr;
  switch (lmax) {
    case 1: kern = pick(std::integral_constant<int, 1>{}); break;
    case 2: kern = pick(std::integral_constant<int, 2>{}); break;
    case 3: kern = pick(std::integral_constant<int, 3>{}); break;
    default: return EGAT_ERR_UNSUPPORTED;
  }
  if (shmem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shmem)) !=
          cudaSuccess)
    return EGAT_ERR_CUDA;
  kern<<<p.plan.tiles, kPlanThreads, shmem, st>>>(p);
  if (lmax >= 3 && cudaGetLastError() == cudaSuccess) {
    const long long slots = (long long)p.plan.tiles * kTileM;
    tile_records_kernel<3><<<unsigned((slots + kRecThreads - 1) / kRecThreads), kRecThreads, 0, st>>>(
        d_order, d_pos, n, p.plan.tiles, p.plan.rec);
  }
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
