// Step 1: cell-list radius graph, exact in integer arithmetic.
//
// [EX] = "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构": §5.1 sets the
// edge cutoff, §5.2 asks for a verified neighbour list.  The plainest exact
// reading: j != i is a neighbour of i iff |p_j - p_i|^2 <= r_c^2 on integer
// grid coordinates; a padded list keeps the K nearest, ties to smaller j.
//
// Design (B200): cells of edge r_c / 2 are mapped to a power-of-two bucket table
// by the Morton code of the low bits of their coordinates, so scratch memory
// depends only on n and the bucket order is a space-filling-curve order.
// Kernels: assign cells -> histogram -> exclusive scan -> scatter -> rank
// atoms inside their bucket by index (deterministic order) -> one warp per atom
// sweeps the 125 surrounding cells, writes the row and counts (padded), or
// counts, scans and writes (CSR).  Rows with more than K neighbours keep the K
// nearest, ranked on the (d^2, j) key.  No kernel waits on another
// block; every loop is bounded.
#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kFillWarps = 4;
constexpr int kSelectCap = 1024;   // neighbour keys a warp can hold in shared memory

struct GraphWs {
  int4* cell;          // [n] (cx, cy, cz, bucket)
  int4* spos;          // [n] bucket-sorted (x, y, z, atom), atoms of a bucket by index
  int4* scell;         // [n] bucket-sorted (cx, cy, cz, 0)
  int4* tpos;          // [n] bucket-sorted in arrival order (before ranking)
  int* bucket_cnt;     // [M]
  int* bucket_start;   // [M + 1]
  int* cursor;         // [M]
  int* deg;            // [n] untruncated degree
  int* trunc;          // [1 + n]: count, then sorted slots of rows with > K neighbours
  int* partial;        // scan partials
  size_t bytes;
};

constexpr int kScanTile = 4096;  // elements per scan block (1024 threads x 4)

int bucket_bits(int n) {
  // bits per axis b, table size M = 2^(3b) >= n, 3 <= b <= 8 (2^b >= 5
  // keeps the 5 x 5 x 5 cells around any cell in distinct buckets).  With
  // several atoms per cell, at least n buckets leave most cells a bucket of
  // their own; atoms of other cells that share a bucket fail the distance
  // test.
  int b = 3;
  while (b < 8 && (int64_t(1) << (3 * b)) < int64_t(n)) ++b;
  return b;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

GraphWs carve(void* base, int n) {
  const int b = bucket_bits(n);
  const size_t M = size_t(1) << (3 * b);
  const size_t nparts = (std::max<size_t>(M + 1, size_t(n) + 1) + kScanTile - 1) / kScanTile;
  GraphWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = static_cast<char*>(base) + off;
    off += align256(bytes);
    return static_cast<void*>(p);
  };
  w.cell = static_cast<int4*>(take(sizeof(int4) * size_t(n)));
  w.spos = static_cast<int4*>(take(sizeof(int4) * size_t(n)));
  w.scell = static_cast<int4*>(take(sizeof(int4) * size_t(n)));
  w.tpos = static_cast<int4*>(take(sizeof(int4) * size_t(n)));
  w.bucket_cnt = static_cast<int*>(take(sizeof(int) * M));
  w.bucket_start = static_cast<int*>(take(sizeof(int) * (M + 1)));
  w.cursor = static_cast<int*>(take(sizeof(int) * M));
  w.deg = static_cast<int*>(take(sizeof(int) * size_t(n)));
  w.trunc = static_cast<int*>(take(sizeof(int) * (size_t(n) + 1)));
  w.partial = static_cast<int*>(take(sizeof(int) * (nparts + 1)));
  w.bytes = off;
  return w;
}

__device__ __forceinline__ int floor_div(int a, int b) {
  // b > 0
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}

__device__ __forceinline__ uint32_t spread3(uint32_t v) {
  // spread the low 8 bits of v to every third bit
  v &= 0xffu;
  v = (v | (v << 8)) & 0x0300f00fu;
  v = (v | (v << 4)) & 0x030c30c3u;
  v = (v | (v << 2)) & 0x09249249u;
  return v;
}

__device__ __forceinline__ int bucket_of(int cx, int cy, int cz, int bits) {
  const uint32_t mask = (1u << bits) - 1u;
  return int(spread3(uint32_t(cx) & mask) | (spread3(uint32_t(cy) & mask) << 1) |
             (spread3(uint32_t(cz) & mask) << 2));
}

__global__ void assign_cells(const int32_t* __restrict__ pos, int n, int cq, int bits,
                             int4* __restrict__ cell, int* __restrict__ bucket_cnt) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int x = pos[3 * i], y = pos[3 * i + 1], z = pos[3 * i + 2];
  const int cx = floor_div(x, cq), cy = floor_div(y, cq), cz = floor_div(z, cq);
  const int b = bucket_of(cx, cy, cz, bits);
  cell[i] = make_int4(cx, cy, cz, b);
  atomicAdd(&bucket_cnt[b], 1);
}

// ---- exclusive scan of int32 counts (three phases, no inter-block waits) ----
__device__ __forceinline__ int block_exclusive_scan(int v, int* smem_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? smem_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) smem_warp[lane] = s;
  }
  __syncthreads();
  const int before = warp > 0 ? smem_warp[warp - 1] : 0;
  total = smem_warp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before + x - v;
}

__global__ void __launch_bounds__(1024) scan_reduce(const int* __restrict__ in, int n,
                                                    int* __restrict__ partial) {
  __shared__ int sw[32];
  const int base = blockIdx.x * kScanTile + threadIdx.x * 4;
  int s = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) s += (base + e < n) ? in[base + e] : 0;
  int total;
  block_exclusive_scan(s, sw, total);
  if (threadIdx.x == 0) partial[blockIdx.x] = total;
}

__global__ void __launch_bounds__(1024) scan_partials(int* __restrict__ partial, int nb) {
  __shared__ int sw[32];
  int carry = 0;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = i < nb ? partial[i] : 0;
    int total;
    const int ex = block_exclusive_scan(v, sw, total);
    if (i < nb) partial[i] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) partial[nb] = carry;
}

// out[i] = sum_{k<i} in[k] for i in [0, n]; out has n + 1 entries.
__global__ void __launch_bounds__(1024) scan_apply(const int* __restrict__ in, int n,
                                                   const int* __restrict__ partial,
                                                   int* __restrict__ out) {
  __shared__ int sw[32];
  const int base = blockIdx.x * kScanTile + threadIdx.x * 4;
  int v[4];
  int s = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[e] = (base + e < n) ? in[base + e] : 0;
    s += v[e];
  }
  int total;
  int ex = block_exclusive_scan(s, sw, total) + partial[blockIdx.x];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (base + e <= n) out[base + e] = ex;
    ex += v[e];
  }
}

// Up to kScanSingle + 1 entries: one CTA, each thread a contiguous chunk of
// at most 9 (larger arrays take the three-phase scan, whose loads coalesce).
constexpr int kScanSingle = 1 << 13;
__global__ void __launch_bounds__(1024) scan_single(const int* __restrict__ in, int n, int* __restrict__ out) {
  __shared__ int sw[32];
  const int per = (n + 1 + 1023) / 1024;
  const int b0 = threadIdx.x * per;
  int s = 0;
  for (int i = b0; i < b0 + per && i < n; ++i) s += in[i];
  int total;
  int ex = block_exclusive_scan(s, sw, total);
  for (int i = b0; i < b0 + per && i <= n; ++i) {
    out[i] = ex;
    if (i < n) ex += in[i];
  }
}

int launch_scan(const int* in, int n, int* partial, int* out, cudaStream_t st) {
  if (n <= kScanSingle) {
    scan_single<<<1, 1024, 0, st>>>(in, n, out);
    return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
  }
  const int nb = (n + 1 + kScanTile - 1) / kScanTile;
  scan_reduce<<<nb, 1024, 0, st>>>(in, n, partial);
  scan_partials<<<1, 1024, 0, st>>>(partial, nb);
  scan_apply<<<nb, 1024, 0, st>>>(in, n, partial, out);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

// Counting-sort scatter: slots within a bucket are taken in arrival order.
__global__ void scatter_atoms(const int32_t* __restrict__ pos, int n,
                              const int4* __restrict__ cell,
                              const int* __restrict__ bucket_start, int* __restrict__ cursor,
                              int4* __restrict__ tpos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int4 c = cell[i];
  const int slot = bucket_start[c.w] + atomicAdd(&cursor[c.w], 1);
  tpos[slot] = make_int4(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2], i);
}

// Deterministic order inside each bucket: an atom's final slot is the bucket
// start plus the number of atoms of its bucket with a smaller index.
__global__ void rank_in_bucket(int n, const int4* __restrict__ cell,
                               const int* __restrict__ bucket_start,
                               const int4* __restrict__ tpos, int4* __restrict__ spos,
                               int4* __restrict__ scell, int32_t* __restrict__ order) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const int4 me = tpos[k];
  const int4 c = cell[me.w];
  const int beg = bucket_start[c.w], end = bucket_start[c.w + 1];
  int rank = 0;
  for (int t = beg; t < end; ++t) rank += tpos[t].w < me.w ? 1 : 0;
  const int dst = beg + rank;
  spos[dst] = me;
  scell[dst] = make_int4(c.x, c.y, c.z, 0);
  if (order) order[dst] = me.w;
}

// Exact squared distance of two grid points in the same 2-cell neighbourhood:
// the coordinate differences fit in 32 bits (the host bounds the cutoff), so
// each square is one widening 32 x 32 -> 64-bit multiply.
__device__ __forceinline__ long long sq_dist(int4 a, int4 b) {
  const int dx = a.x - b.x, dy = a.y - b.y, dz = a.z - b.z;
  return (long long)dx * dx + (long long)dy * dy + (long long)dz * dz;
}

struct Search {
  const int4* spos;
  const int4* scell;
  const int* bucket_start;
  int bits;
  long long rc2;
  int key_shift;
  int cq;          // cell edge (grid units)
};

// Distance along one axis from coordinate v to the cell c of edge cq, whose
// points have coordinates c*cq .. c*cq + cq - 1 (0 when v lies in it).
__device__ __forceinline__ long long axis_gap(int v, int c, int cq) {
  const long long lo = (long long)c * cq, hi = lo + cq - 1;
  return v < lo ? lo - v : (v > hi ? v - hi : 0);
}

// Cells have edge ceil(r_c / 2), so every neighbour lies in the 5 x 5 x 5
// block of cells around the atom's cell.
constexpr int kSpan = 2;
constexpr int kWidth = 2 * kSpan + 1;
constexpr int kBlockCells = kWidth * kWidth * kWidth;

// Visit every candidate of atom p (cell c) once; f(hit, j, d2) is called by
// every lane of the warp together (full-warp ballots are allowed inside), hit
// marking a neighbour within the cutoff.  Cells are taken 32 at a time: each
// lane loads one cell's bucket range, a warp scan lays the ranges end to end,
// and the warp walks that flat candidate list 32 at a time, each lane finding
// its candidate's cell by a binary search over the scanned offsets.  Warps
// that share a sweep take rounds round0, round0 + round_step, ... and, within
// a round, candidate chunks part, part + parts, ...
template <typename F>
__device__ __forceinline__ void for_each_neighbour_rounds(const Search& s, int4 p, int4 c,
                                                          int round0, int round_step, int part,
                                                          int parts, F&& f) {
  const int lane = threadIdx.x & 31;
  for (int r0 = round0 * 32; r0 < kBlockCells; r0 += round_step * 32) {
    const int l = r0 + lane;
    int beg = 0, len = 0, cx = 0, cy = 0, cz = 0;
    if (l < kBlockCells) {
      cx = c.x + l % kWidth - kSpan;
      cy = c.y + (l / kWidth) % kWidth - kSpan;
      cz = c.z + l / (kWidth * kWidth) - kSpan;
      // a cell whose box lies beyond the cutoff from p holds no neighbour
      const long long gx = axis_gap(p.x, cx, s.cq), gy = axis_gap(p.y, cy, s.cq),
                      gz = axis_gap(p.z, cz, s.cq);
      if (gx * gx + gy * gy + gz * gz <= s.rc2) {
        const int b = bucket_of(cx, cy, cz, s.bits);
        beg = s.bucket_start[b];
        len = s.bucket_start[b + 1] - beg;
      }
    }
    int inc = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const int total = __shfl_sync(0xffffffffu, inc, 31);
    const int exc = inc - len;
    for (int base = part * 32; base < total; base += parts * 32) {
      const int k = base + lane;
      // owner: the last lane whose range starts at or before k
      int own = 0;
#pragma unroll
      for (int step = 16; step > 0; step >>= 1) {
        const int e = __shfl_sync(0xffffffffu, exc, own + step);
        if (e <= k) own += step;
      }
      const int obeg = __shfl_sync(0xffffffffu, beg, own);
      const int oexc = __shfl_sync(0xffffffffu, exc, own);
      bool hit = false;
      int j = -1;
      long long d2 = 0;
      if (k < total) {
        // A bucket may also hold atoms of cells outside the 5 x 5 x 5 block
        // (their low coordinate bits collide).  Such an atom is at least
        // 2 cq + 1 > r_c away along one axis, so the cutoff test rejects it
        // and the cell itself needs no check.
        const int4 q = s.spos[obeg + (k - oexc)];
        j = q.w;
        d2 = sq_dist(q, p);
        hit = (j != p.w) && (d2 <= s.rc2);
      }
      f(hit, j, d2);
    }
  }
}

template <typename F>
__device__ __forceinline__ void for_each_neighbour(const Search& s, int4 p, int4 c, F&& f) {
  for_each_neighbour_rounds(s, p, c, 0, 1, 0, 1, f);
}

__global__ void count_neighbours(Search s, int n, int* __restrict__ deg) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= n) return;
  const int4 p = s.spos[w];
  const int4 c = s.scell[w];
  int cnt = 0;
  for_each_neighbour(s, p, c, [&](bool hit, int, long long) { cnt += hit ? 1 : 0; });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) deg[p.w] = cnt;
}

// K-th smallest key (d^2 << shift | j) among the atom's neighbours, by
// bisection over the key range; every key is distinct because j is.
__device__ unsigned long long kth_key(const Search& s, int4 p, int4 c, int K) {
  const unsigned long long jmask = (1ull << s.key_shift) - 1ull;
  unsigned long long lo = 0, hi = ((unsigned long long)s.rc2 << s.key_shift) | jmask;
  while (lo < hi) {
    const unsigned long long mid = lo + ((hi - lo) >> 1);
    int cnt = 0;
    for_each_neighbour(s, p, c, [&](bool hit, int j, long long d2) {
      cnt += (hit && ((((unsigned long long)d2) << s.key_shift) | (unsigned long long)j) <= mid)
                 ? 1 : 0;
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= K) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Padded list, one warp per atom (atoms taken in cell order).  One sweep
// writes the first K neighbours and counts all of them; an atom with more
// than K is appended to the truncation list for fix_truncated.  Row order is
// the sweep order: the 125 cells in a fixed order, atoms of a cell by index —
// deterministic, independent of thread scheduling.
__global__ void __launch_bounds__(kFillWarps * 32, 12)
fill_padded(Search s, int n, int K, int32_t* __restrict__ nbr, int32_t* __restrict__ cnt,
            int* __restrict__ trunc) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kFillWarps + (threadIdx.x >> 5);
  if (w >= n) return;
  const int4 p = s.spos[w];
  const int4 c = s.scell[w];
  int32_t* row = nbr + (long long)p.w * K;
  int total = 0;
  for_each_neighbour(s, p, c, [&](bool hit, int j, long long) {
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    const int pos = total + __popc(m & ((1u << lane) - 1u));
    if (hit && pos < K) row[pos] = j;
    total += __popc(m);
  });
  const int take = total < K ? total : K;
  for (int t = take + lane; t < K; t += 32) row[t] = -1;
  if (lane == 0) {
    cnt[p.w] = take;
    if (total > K) trunc[1 + atomicAdd(&trunc[0], 1)] = w;
  }
}

// Rows with more than K neighbours: one CTA of kFixWarps warps per listed atom
// (persistent CTAs; the loop is bounded by the device-side count).  The warps
// split the 125-cell sweep (four rounds of 32 cells, each round's candidates
// in kFixWarps / 4 interleaved parts) and gather every neighbour's key
// (d^2 << shift | j) into shared memory.  The keys are distinct (j is), so a
// key's rank among them is its place in the row: the key of rank r < K writes
// row[r], and the row lists the K nearest, nearest first, ties to the smaller
// index.  A row with more keys than the buffer holds first finds its K-th
// smallest key by bisection (one warp), then gathers the K keys up to it and
// ranks those.
constexpr int kFixWarps = 16;
constexpr int kFixRounds = (kBlockCells + 31) / 32;
static_assert(kFixWarps % kFixRounds == 0, "whole rounds per group of warps");

__global__ void __launch_bounds__(kFixWarps * 32)
fix_truncated(Search s, int K, int32_t* __restrict__ nbr, const int* __restrict__ trunc,
              int* __restrict__ overflow) {
  __shared__ unsigned long long keys[kSelectCap];
  __shared__ unsigned long long s_thresh;
  __shared__ int s_total, s_kept;
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int ntr = trunc[0];
  const unsigned long long jmask = (1ull << s.key_shift) - 1ull;
  // every warp sweeps its rounds of cells; f(hit, key) with full-warp ballots
  auto gather = [&](const int4& p, const int4& c, int* counter, auto keep) {
    for_each_neighbour_rounds(s, p, c, wib % kFixRounds, kFixRounds, wib / kFixRounds,
                              kFixWarps / kFixRounds, [&](bool hit, int j, long long d2) {
      const unsigned long long key = (((unsigned long long)d2) << s.key_shift) | (unsigned long long)j;
      const bool take = hit && keep(key);
      const unsigned m = __ballot_sync(0xffffffffu, take);
      int base = 0;
      if (lane == 0 && m) base = atomicAdd(counter, __popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int pos = base + __popc(m & ((1u << lane) - 1u));
      if (take && pos < kSelectCap) keys[pos] = key;
    });
  };
  for (int t = blockIdx.x; t < ntr; t += gridDim.x) {
    const int w = trunc[1 + t];
    const int4 p = s.spos[w];
    const int4 c = s.scell[w];
    int32_t* row = nbr + (long long)p.w * K;
    if (threadIdx.x == 0) {
      s_total = 0;
      s_kept = 0;
    }
    __syncthreads();
    gather(p, c, &s_total, [](unsigned long long) { return true; });
    __syncthreads();
    const int total = s_total;
    int T = total;
    if (total > kSelectCap) {
      if (wib == 0) {
        const unsigned long long th = kth_key(s, p, c, K);
        if (lane == 0) s_thresh = th;
      }
      __syncthreads();
      const unsigned long long th = s_thresh;
      gather(p, c, &s_kept, [th](unsigned long long key) { return key <= th; });
      __syncthreads();
      T = s_kept < kSelectCap ? s_kept : kSelectCap;   // K of them
    }
    for (int i = threadIdx.x; i < T; i += blockDim.x) {
      const unsigned long long key = keys[i];
      int rank = 0;
#pragma unroll 4
      for (int k = 0; k < T; ++k) rank += keys[k] < key ? 1 : 0;
      if (rank < K) row[rank] = int32_t(key & jmask);
    }
    if (threadIdx.x == 0) atomicAdd(overflow, total - K);
    __syncthreads();
  }
}

// CSR rows (after count_neighbours and the scan): every neighbour, in sweep order.
__global__ void __launch_bounds__(kFillWarps * 32)
fill_csr(Search s, int n, const int* __restrict__ rowptr, int32_t* __restrict__ col,
         long long col_capacity, int* __restrict__ overflow) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kFillWarps + (threadIdx.x >> 5);
  if (w >= n) return;
  const int4 p = s.spos[w];
  const int4 c = s.scell[w];
  const long long base = rowptr[p.w];
  int written = 0;
  for_each_neighbour(s, p, c, [&](bool hit, int j, long long) {
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    const long long pos = base + written + __popc(m & ((1u << lane) - 1u));
    if (hit && pos < col_capacity) col[pos] = j;
    written += __popc(m);
  });
  if (lane == 0 && base + written > col_capacity)
    atomicAdd(overflow, int(base >= col_capacity ? (long long)written
                                                 : base + written - col_capacity));
}

}  // namespace

size_t graph_workspace_bytes(int n) { return carve(nullptr, n).bytes; }

int build_graph(const int32_t* d_pos_q, int n, int cutoff_q, int K, int mode,
                int32_t* d_a, int32_t* d_b, long long col_capacity, int32_t* d_order,
                int32_t* d_overflow, void* d_ws, size_t ws_bytes, cudaStream_t st) {
  GraphWs w = carve(d_ws, n);
  if (ws_bytes < w.bytes) return EGAT_ERR_WORKSPACE;
  const int bits = bucket_bits(n);
  const int M = 1 << (3 * bits);
  int key_shift = 1;
  while ((1ll << key_shift) < n) ++key_shift;

  if (cudaMemsetAsync(d_overflow, 0, sizeof(int32_t), st) != cudaSuccess) return EGAT_ERR_CUDA;
  if (cudaMemsetAsync(w.bucket_cnt, 0, sizeof(int) * M, st) != cudaSuccess) return EGAT_ERR_CUDA;
  if (cudaMemsetAsync(w.cursor, 0, sizeof(int) * M, st) != cudaSuccess) return EGAT_ERR_CUDA;

  const int tb = 256;
  const unsigned nb = unsigned((n + tb - 1) / tb);
  const int cell_q = (cutoff_q + 1) / 2;   // cell edge ceil(r_c / 2)
  assign_cells<<<nb, tb, 0, st>>>(d_pos_q, n, cell_q, bits, w.cell, w.bucket_cnt);
  if (launch_scan(w.bucket_cnt, M, w.partial, w.bucket_start, st) != EGAT_OK) return EGAT_ERR_CUDA;
  scatter_atoms<<<nb, tb, 0, st>>>(d_pos_q, n, w.cell, w.bucket_start, w.cursor, w.tpos);
  rank_in_bucket<<<nb, tb, 0, st>>>(n, w.cell, w.bucket_start, w.tpos, w.spos, w.scell, d_order);
  Search s{w.spos, w.scell, w.bucket_start, bits, (long long)cutoff_q * cutoff_q, key_shift, cell_q};
  const unsigned nfill = unsigned((n + kFillWarps - 1) / kFillWarps);
  if (mode == EGAT_GRAPH_PADDED) {
    if (cudaMemsetAsync(w.trunc, 0, sizeof(int), st) != cudaSuccess) return EGAT_ERR_CUDA;
    fill_padded<<<nfill, kFillWarps * 32, 0, st>>>(s, n, K, d_a, d_b, w.trunc);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    fix_truncated<<<sms * 4, kFixWarps * 32, 0, st>>>(s, K, d_a, w.trunc, d_overflow);
  } else {
    const long long nthreads = (long long)n * 32;
    count_neighbours<<<unsigned((nthreads + tb - 1) / tb), tb, 0, st>>>(s, n, w.deg);
    if (launch_scan(w.deg, n, w.partial, d_a, st) != EGAT_OK) return EGAT_ERR_CUDA;
    fill_csr<<<nfill, kFillWarps * 32, 0, st>>>(s, n, d_a, d_b, col_capacity, d_overflow);
  }
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
