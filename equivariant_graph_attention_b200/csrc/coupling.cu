// Step 2: EAAS source coupling h'_j = h_j (x) R(r_j).
//
// [EX] = "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §2.1-§2.3
// (alignment rotation, sparse re-index, Proposition 4.3), §3.1 step 1;
// [TS] = "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
// Memory" §2.1 (Lemma 4.1: only m = 0 of the solid harmonic survives in the
// aligned frame; Eq. 13: the re-index rule).
//
// Kernel layout: a group of C/CPL lanes per atom, each lane owning CPL
// consecutive channels.  The group builds the atom's Wigner-D matrices
// (degree 1 from the alignment rotation, higher degrees by the
// Ivanic–Ruedenberg recursion, entries in parallel) in shared memory once;
// each lane then rotates its channels' components into the aligned frame,
// applies the sparse re-index with the path weights, and rotates back.
// Memory traffic is one read of h and one write of h' (streaming, HBM-bound).
#include <cmath>
#include <mutex>

#include "egat_async.cuh"
#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {

// ---------------------------------------------------------------------------
// host: Clebsch–Gordan coefficients and the re-index table
// ---------------------------------------------------------------------------
double clebsch_gordan(int j1, int m1, int j2, int m2, int J, int M) {
  if (M != m1 + m2) return 0.0;
  if (J < std::abs(j1 - j2) || J > j1 + j2) return 0.0;
  if (std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0.0;
  auto f = [](int k) {
    double r = 1.0;
    for (int t = 2; t <= k; ++t) r *= t;
    return r;
  };
  const double pre = (2.0 * J + 1.0) * f(J + j1 - j2) * f(J - j1 + j2) * f(j1 + j2 - J) /
                     f(j1 + j2 + J + 1) * f(J + M) * f(J - M) * f(j1 - m1) * f(j1 + m1) *
                     f(j2 - m2) * f(j2 + m2);
  double sum = 0.0;
  for (int k = 0; k <= j1 + j2 - J; ++k) {
    const int a[6] = {k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k,
                      J - j1 - m2 + k};
    bool ok = true;
    for (int t = 0; t < 6; ++t) ok = ok && a[t] >= 0;
    if (!ok) continue;
    double den = 1.0;
    for (int t = 0; t < 6; ++t) den *= f(a[t]);
    sum += ((k & 1) ? -1.0 : 1.0) / den;
  }
  return std::sqrt(pre) * sum;
}

namespace {
EaasTable g_tables[kMaxL + 1];
std::once_flag g_table_once;

void fill_tables() {
  for (int L = 1; L <= kMaxL; ++L) {
    EaasTable& t = g_tables[L];
    for (int p = 0; p < kMaxPaths; ++p)
      for (int m = 0; m < 2 * kMaxL + 1; ++m) t.f[p][m] = 0.f;
    const int np = num_paths(L);
    for (int p = 0; p < np; ++p) {
      const int li = path_info(L, p, 0), lf = path_info(L, p, 1), lo = path_info(L, p, 2);
      const bool even = ((li + lf + lo) % 2) == 0;
      for (int mo = -lo; mo <= lo; ++mo) {
        double v = 0.0;
        if (std::abs(mo) <= li) {
          if (even) {
            // m_i = m_o: <li m; lf 0 | lo m>
            v = clebsch_gordan(li, mo, lf, 0, lo, mo);
          } else if (mo != 0) {
            // m_i = -m_o: sgn(m_o) <li |m|; lf 0 | lo |m|>
            const int am = std::abs(mo);
            v = (mo > 0 ? 1.0 : -1.0) * clebsch_gordan(li, am, lf, 0, lo, am);
          }
        }
        t.f[p][mo + lo] = float(v);
      }
    }
  }
}
}  // namespace

const EaasTable& eaas_table(int L) {
  std::call_once(g_table_once, fill_tables);
  return g_tables[L];
}

// ---------------------------------------------------------------------------
// device: source coupling kernel
// ---------------------------------------------------------------------------
namespace {

constexpr int kEaasWarps = 8;

struct EaasParams {
  const void* x;
  const float* pos;
  const float* w;
  void* y;
  int n;
  int C;
  const float* rec;   // planned form: the attention plan's tile records
  long long items;    // atoms, or target slots of the plan (tiles * kTileM)
  EaasTable tab;
};

// CPL consecutive channels of one component row (vector load / store).
template <typename T, int CPL>
struct ChanVec;
template <>
struct ChanVec<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[4]) {
    unpack(__ldg(reinterpret_cast<const uint2*>(p)), v);
  }
  static __device__ __forceinline__ void load_shared(const __nv_bfloat16* p, float (&v)[4]) {
    unpack(*reinterpret_cast<const uint2*>(p), v);
  }
  static __device__ __forceinline__ void unpack(const uint2 u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};
template <>
struct ChanVec<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[2]) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xffff0000u);
  }
  static __device__ __forceinline__ void load_shared(const __nv_bfloat16* p, float (&v)[2]) {
    const uint32_t u = *reinterpret_cast<const unsigned int*>(p);
    v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xffff0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[2]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    *reinterpret_cast<__nv_bfloat162*>(p) = a;
  }
};
template <>
struct ChanVec<float, 4> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void load_shared(const float* p, float (&v)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <>
struct ChanVec<float, 2> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[2]) {
    const float2 u = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = u.x; v[1] = u.y;
  }
  static __device__ __forceinline__ void load_shared(const float* p, float (&v)[2]) {
    const float2 u = *reinterpret_cast<const float2*>(p);
    v[0] = u.x; v[1] = u.y;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  }
};

// float32 stores rounded to tf32 (round to nearest, ties away): the operand
// format of the backward's tf32 products, so they read the bits unconverted.
// One float wide, so that pointer arithmetic on it steps in floats.
struct Tf32Out {
  float v;
};
static_assert(sizeof(Tf32Out) == sizeof(float) && alignof(Tf32Out) == alignof(float), "Tf32Out is a float");
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
template <int N>
struct ChanVec<Tf32Out, N> {
  static __device__ __forceinline__ void store(Tf32Out* p, const float (&v)[N]) {
    float w[N];
#pragma unroll
    for (int e = 0; e < N; ++e) w[e] = round_tf32(v[e]);
    ChanVec<float, N>::store(reinterpret_cast<float*>(p), w);
  }
};

// A group of G = C/CPL lanes owns one atom; each lane owns CPL consecutive
// channels (CPL = 4 up to lmax 2, 2 at lmax 3 for the register budget), so
// component rows move in 8-16 byte vectors.  The group builds the atom's
// Wigner-D matrices once in shared memory (groups of up to 32 lanes inside a
// warp; a 64-lane group spans two warps, each building its own copy), then
// every lane couples its channels with the matrices held in registers.
// PLANNED: the items are the target slots of an attention plan, whose tile
// records already hold each atom's index, |r|^l and Wigner-D matrices; the
// group copies them instead of building them.
template <int L, typename T, bool PLANNED, typename TO = T>
__global__ void __launch_bounds__(kEaasWarps * 32, (L >= 3 ? 1 : 2))
eaas_source_kernel(const __grid_constant__ EaasParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int WS = wig_size(L);
  constexpr int CPL = L >= 3 ? 2 : 4;
  constexpr int kMaxSlots = 32 / 4;              // C >= 16 -> G >= 4 lanes
  constexpr int NP = num_paths(L);
  __shared__ float Dsm[kEaasWarps][kMaxSlots][WS];
  extern __shared__ float sw[];                   // path weights [P][C]

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int C = p.C;
  const int G = C / CPL;                        // lanes per atom
  const int WPA = G > 32 ? G / 32 : 1;          // warps per atom
  const int GW = G > 32 ? 32 : G;               // lanes of this warp in the group
  const int AW = 32 / GW;                       // atoms per warp
  const int slot = lane / GW;
  const int gl = lane % GW;                     // lane within the warp's part of the group
  const long long gwarp = (long long)blockIdx.x * kEaasWarps + wib;
  const long long nwarps = (long long)gridDim.x * kEaasWarps;
  const int part = int(gwarp % WPA);            // which warp of the atom's group
  const int c0 = (part * 32 + gl) * CPL;         // first channel of this lane
  const long long ngroups = (p.items + AW - 1) / AW;
  constexpr int REC = plan_record_words(L);
  const T* __restrict__ x = static_cast<const T*>(p.x);
  TO* __restrict__ y = static_cast<TO*>(p.y);
  float* Dme = Dsm[wib][slot];
  for (int e = threadIdx.x; e < NP * C; e += blockDim.x) sw[e] = __ldg(p.w + e);
  __syncthreads();

  for (long long grp = gwarp / WPA; grp < ngroups; grp += nwarps / WPA) {
    const long long item = grp * AW + slot;
    long long at = item;
    bool live = item < p.items;
    const float* R = nullptr;
    int rs = 0;
    if constexpr (PLANNED) {
      if (live) {
        R = p.rec + (item / kTileM) * REC;
        rs = int(item % kTileM);
        at = reinterpret_cast<const int*>(R)[kRecTgt + rs];
        live = (unsigned long long)at < (unsigned long long)p.n;
      }
    }
    float Q[9];
    float r = 0.f;
    if constexpr (!PLANNED) {
      if (live) r = alignment_rotation(__ldg(p.pos + 3 * at), __ldg(p.pos + 3 * at + 1),
                                       __ldg(p.pos + 3 * at + 2), Q);
      else alignment_rotation(0.f, 0.f, 0.f, Q);
    }
    float xv[CPL][D];
    if (live) {
      const T* xr = x + (size_t)at * D * C + c0;
#pragma unroll
      for (int d = 0; d < D; ++d) {
        float v[CPL];
        ChanVec<T, CPL>::load(xr + d * C, v);
#pragma unroll
        for (int k = 0; k < CPL; ++k) xv[k][d] = v[k];
      }
    }
    float rpow[L + 1];
    if constexpr (PLANNED) {
#pragma unroll
      for (int l = 0; l <= L; ++l) rpow[l] = live ? __ldg(R + kRecRp + rs * (L + 1) + l) : 0.f;
      __syncwarp();                           // previous atom's readers are done
      if (live)
        for (int e = gl; e < WS; e += GW) Dme[e] = __ldg(R + rec_off_D(L) + rs * WS + e);
      __syncwarp();
    } else {
      rpow[0] = 1.f;
#pragma unroll
      for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
      __syncwarp();                           // previous atom's readers are done
      wigner_build<L>(Q, Dme, gl, GW, [] { __syncwarp(); });
    }
    if (live) {
      TO* yr = y + (size_t)at * D * C + c0;
      const float* swc = sw + c0;
      eaas_multi<L, CPL>(xv, Dme, rpow, p.tab, [&](int q, int k) { return swc[q * C + k]; },
                         [&](int d, const float (&v)[CPL]) { ChanVec<TO, CPL>::store(yr + d * C, v); });
    }
  }
}
// Planned source coupling staged by tiles, for C = 128 (up to lmax 2, and
// lmax 3 in bf16, each slot in two channel halves).  Persistent CTAs of
// kTileM / 2 warps (two per SM up to lmax 2) take the plan's tiles in turn.
// The tile record arrives by one bulk copy two tiles ahead and the tile's 16
// feature rows by 16 bulk copies one tile ahead (double-buffered), so the
// loads stream while the previous tile is coupled; warp w couples target
// slots w and w + kTileM / 2 from shared memory (rotation and |r|^l from the
// record) and writes their h' rows (in TO) straight to global memory.  A
// warp done with a tile arrives on that tile's done mbarrier; warp 0 refills
// a buffer once all warps have arrived, so warps never wait on a block
// barrier.  Every wait is bounded.
template <int L, typename T>
struct TileSmem {
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int CPL = L >= 3 ? 2 : 4;    // channels per lane in one pass over a slot
  static constexpr int C = 128;
  static constexpr int HALVES = C / (32 * CPL); // passes per slot (2 at lmax 3)
  static constexpr int ROWB = D * C * int(sizeof(T));
  static constexpr int REC = plan_record_words(L);
  static constexpr size_t rows = 0;                                       // [2][16][ROWB]
  static constexpr size_t recs = rows + size_t(2) * kTileM * ROWB;        // [3][REC]
  static constexpr size_t sw = recs + size_t(3) * REC * 4;                // [P][C]
  static constexpr size_t bars = sw + size_t(num_paths(L)) * C * 4;       // rows [2], records [3], consumed [2]
  static constexpr size_t total = bars + 7 * 8 + 16;
  static_assert(ROWB % 16 == 0 && REC % 4 == 0 && bars % 8 == 0, "bulk-copy alignment");
};

// half a tile's warps per CTA, two CTAs per SM (one at lmax 3, whose rows
// fill the shared memory)
constexpr int kHalfWarps = kTileM / 2;
template <int L, typename T, typename TO = T>
__global__ void __launch_bounds__(kHalfWarps * 32, L >= 3 ? 1 : 2)
eaas_tile_kernel(const __grid_constant__ EaasParams p) {
  using Sm = TileSmem<L, T>;
  constexpr int D = Sm::D, CPL = Sm::CPL, C = Sm::C, ROWB = Sm::ROWB, REC = Sm::REC;
  constexpr int HALVES = Sm::HALVES;
  constexpr int WS = wig_size(L);
  constexpr int NP = num_paths(L);
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* rows = smem + Sm::rows;
  float* recs = reinterpret_cast<float*>(smem + Sm::recs);
  float* sw = reinterpret_cast<float*>(smem + Sm::sw);
  uint64_t* rowbar = reinterpret_cast<uint64_t*>(smem + Sm::bars);   // [2] a tile's rows
  uint64_t* recbar = rowbar + 2;                                     // [3] a tile record
  uint64_t* donebar = recbar + 3;                                    // [2] every warp done with a tile
  volatile int* abort_flag = reinterpret_cast<volatile int*>(donebar + 2);

  const int tid = threadIdx.x, lane = tid & 31, wfirst = tid >> 5;
  const int tiles = int(p.items / kTileM);
  const int grid = gridDim.x;
  if (blockIdx.x >= tiles) return;   // whole CTA
  if (tid == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(smem_u32(rowbar + b), 1);
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(donebar + b), kHalfWarps);
    mbar_fence_init();
    *abort_flag = 0;
  }
  for (int e = tid; e < NP * C; e += blockDim.x) sw[e] = __ldg(p.w + e);
  __syncthreads();

  const char* xb = static_cast<const char*>(p.x);
  TO* __restrict__ y = static_cast<TO*>(p.y);
  // thread 0: a tile's record into recs[b]
  auto issue_rec = [&](int tl, int b) {
    const uint32_t bar = smem_u32(recbar + b);
    mbar_arrive_expect_tx(bar, REC * 4);
    bulk_g2s(smem_u32(recs + b * REC), p.rec + (long long)tl * REC, REC * 4, bar);
  };
  // thread 0: the feature rows of a tile's targets into rows[b] (empty slots
  // are not copied); used for the first tile, warp 0 issues the later ones
  auto issue_rows = [&](const float* rec, int b) {
    const int* tg = reinterpret_cast<const int*>(rec) + kRecTgt;
    int valid = 0;
    for (int r = 0; r < kTileM; ++r) valid += (unsigned)tg[r] < (unsigned)p.n;
    const uint32_t bar = smem_u32(rowbar + b);
    mbar_arrive_expect_tx(bar, uint32_t(valid) * ROWB);
    for (int r = 0; r < kTileM; ++r)
      if ((unsigned)tg[r] < (unsigned)p.n)
        bulk_g2s(smem_u32(rows + (size_t(b) * kTileM + r) * ROWB), xb + (size_t)tg[r] * ROWB, ROWB,
                 bar);
  };

  int tile = blockIdx.x;
  if (tid == 0) {
    issue_rec(tile, 0);
    bounded_wait(smem_u32(recbar), 0u, kWaitPolls, abort_flag);
    issue_rows(recs, 0);
    if (tile + grid < tiles) issue_rec(tile + grid, 1);
  }
  int j = 0;   // this CTA's tile sequence number
  for (; tile < tiles; ++j, tile += grid) {
    const int rb = j % 3, wb = j & 1;
    bounded_wait(smem_u32(recbar + rb), uint32_t(j / 3) & 1u, kWaitPolls, abort_flag);
    bounded_wait(smem_u32(rowbar + wb), uint32_t(j >> 1) & 1u, kWaitPolls, abort_flag);
    if (wfirst == 0 && tile + grid < tiles) {
      // warp 0: the next tile's rows (its record arrived a tile ago), one
      // bulk copy per lane after lane 0 has announced their bytes, and the
      // record after it; both buffers were last read by tile j - 1, which
      // every warp has signalled done on donebar[(j - 1) & 1]
      if (j >= 1)
        bounded_wait(smem_u32(donebar + ((j + 1) & 1)), uint32_t((j - 1) >> 1) & 1u, kWaitPolls, abort_flag);
      const int nb = (j + 1) % 3;
      bounded_wait(smem_u32(recbar + nb), uint32_t((j + 1) / 3) & 1u, kWaitPolls, abort_flag);
      const int* tg = reinterpret_cast<const int*>(recs + nb * REC) + kRecTgt;
      const int wbn = (j + 1) & 1;
      const uint32_t bar = smem_u32(rowbar + wbn);
      const bool mine = lane < kTileM && (unsigned)tg[lane < kTileM ? lane : 0] < (unsigned)p.n;
      const int valid = __popc(__ballot_sync(0xffffffffu, mine));
      if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(valid) * ROWB);
      __syncwarp();
      if (mine)
        bulk_g2s(smem_u32(rows + (size_t(wbn) * kTileM + lane) * ROWB), xb + (size_t)tg[lane] * ROWB,
                 ROWB, bar);
      if (lane == 0 && tile + 2 * grid < tiles) issue_rec(tile + 2 * grid, (j + 2) % 3);
    }
    const float* rec = recs + rb * REC;
    for (int w = wfirst; w < kTileM; w += kHalfWarps) {   // two slots per warp
    const int at = reinterpret_cast<const int*>(rec)[kRecTgt + w];
    if ((unsigned)at < (unsigned)p.n) {
      float rpow[L + 1];
#pragma unroll
      for (int l = 0; l <= L; ++l) rpow[l] = rec[kRecRp + w * (L + 1) + l];
#pragma unroll 1
      for (int hf = 0; hf < HALVES; ++hf) {
        const int c0 = (hf * 32 + lane) * CPL;   // this lane's first channel in this pass
        const T* xr = reinterpret_cast<const T*>(rows + (size_t(wb) * kTileM + w) * ROWB) + c0;
        float xv[CPL][D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
          float v[CPL];
          ChanVec<T, CPL>::load_shared(xr + d * C, v);
#pragma unroll
          for (int k = 0; k < CPL; ++k) xv[k][d] = v[k];
        }
        TO* yr = y + (size_t)at * D * C + c0;
        const float* swc = sw + c0;
        eaas_multi<L, CPL, (CPL >= 4)>(xv, rec + rec_off_D(L) + w * WS, rpow, p.tab,
                           [&](int q, int k) { return swc[q * C + k]; },
                           [&](int d, const float (&v)[CPL]) { ChanVec<TO, CPL>::store(yr + d * C, v); });
      }
    }
    }
    // this warp is done with rows[wb] and recs[rb]: warp 0 refills them one
    // and two tiles ahead once every warp has said so (no block barrier, so
    // a warp that finishes early starts the next tile)
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(donebar + wb));
  }
  if (*abort_flag && tid == 0) {
    // a wait gave up: give every barrier's last phase a short, bounded chance
    // to complete before the CTA's shared memory is released
    volatile int none = 0;
    for (int b = 0; b < 2; ++b) {
      const int last = j - 1 - ((j - 1 - b) & 1);   // last tile sequence number with j % 2 == b
      if (last >= 0) bounded_wait(smem_u32(rowbar + b), uint32_t(last >> 1) & 1u, kDrainPolls, &none);
    }
    for (int b = 0; b < 3; ++b) {
      int last = j - 1;
      while (last >= 0 && last % 3 != b) --last;
      if (last >= 0) bounded_wait(smem_u32(recbar + b), uint32_t(last / 3) & 1u, kDrainPolls, &none);
    }
  }
}

template <int L, typename T, bool PLANNED, typename TO = T>
int launch_eaas_t(const egat_shape& s, const void* d_x, const float* d_pos, const float* rec,
                  long long items, const float* d_w, void* d_y, cudaStream_t st) {
  EaasParams p;
  p.x = d_x;
  p.pos = d_pos;
  p.w = d_w;
  p.y = d_y;
  p.n = s.n;
  p.C = s.C;
  p.rec = rec;
  p.items = items;
  p.tab = eaas_table(L);
  constexpr int CPL = L >= 3 ? 2 : 4;
  const int G = s.C / CPL;
  const int WPA = G > 32 ? G / 32 : 1;
  const int AW = 32 / (G > 32 ? 32 : G);
  const long long groups = (items + AW - 1) / AW;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (groups * WPA + kEaasWarps - 1) / kEaasWarps;
  const int grid = int(std::max<long long>(1, std::min<long long>(want, (long long)sms * 8)));
  const size_t shmem = size_t(num_paths(L)) * s.C * sizeof(float);
  eaas_source_kernel<L, T, PLANNED, TO><<<grid, kEaasWarps * 32, shmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace

int launch_eaas_source(const egat_shape& s, const void* d_x, const float* d_pos,
                       const float* d_w, void* d_y, cudaStream_t st) {
  const bool bf = s.dtype == EGAT_BF16;
  const long long n = s.n;
  switch (s.lmax) {
    case 1: return bf ? launch_eaas_t<1, __nv_bfloat16, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<1, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    case 2: return bf ? launch_eaas_t<2, __nv_bfloat16, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<2, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    case 3: return bf ? launch_eaas_t<3, __nv_bfloat16, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<3, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

template <int L, typename T, typename TO = T>
int launch_eaas_tile(const egat_shape& s, const void* d_x, const float* rec, long long items,
                     const float* d_w, void* d_y, cudaStream_t st) {
  EaasParams p;
  p.x = d_x;
  p.pos = nullptr;
  p.w = d_w;
  p.y = d_y;
  p.n = s.n;
  p.C = s.C;
  p.rec = rec;
  p.items = items;
  p.tab = eaas_table(L);
  constexpr size_t shmem = TileSmem<L, T>::total;
  auto kern = eaas_tile_kernel<L, T, TO>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shmem)) !=
      cudaSuccess)
    return EGAT_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = int(items / kTileM);
  // two CTAs per SM while two fit in shared memory (lmax <= 2), else one
  const int per_sm = 2 * shmem <= 227 * 1024 ? 2 : 1;
  const int grid = tiles < per_sm * sms ? tiles : per_sm * sms;
  kern<<<grid, kHalfWarps * 32, shmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

int launch_eaas_source_f32out(const egat_shape& s, const void* d_x, const float* d_pos,
                              const float* d_w, float* d_y, cudaStream_t st) {
  const bool bf = s.dtype == EGAT_BF16;
  const long long n = s.n;
  switch (s.lmax) {
    case 1: return bf ? launch_eaas_t<1, __nv_bfloat16, false, float>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<1, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    case 2: return bf ? launch_eaas_t<2, __nv_bfloat16, false, float>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<2, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    case 3: return bf ? launch_eaas_t<3, __nv_bfloat16, false, float>(s, d_x, d_pos, nullptr, n, d_w, d_y, st)
                      : launch_eaas_t<3, float, false>(s, d_x, d_pos, nullptr, n, d_w, d_y, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

int launch_eaas_planned(const egat_shape& s, const void* d_x, const void* d_plan, const float* d_w,
                        void* d_y, cudaStream_t st) {
  const bool bf = s.dtype == EGAT_BF16;
  const PlanView pv = plan_view(const_cast<void*>(d_plan), s.n, s.K, s.lmax);
  const long long items = (long long)pv.tiles * kTileM;
  // one warp per atom: the tile-staged kernel
  if (s.lmax <= 2 && s.C == 128) {
    if (s.lmax == 1) return bf ? launch_eaas_tile<1, __nv_bfloat16>(s, d_x, pv.rec, items, d_w, d_y, st)
                               : launch_eaas_tile<1, float>(s, d_x, pv.rec, items, d_w, d_y, st);
    return bf ? launch_eaas_tile<2, __nv_bfloat16>(s, d_x, pv.rec, items, d_w, d_y, st)
              : launch_eaas_tile<2, float>(s, d_x, pv.rec, items, d_w, d_y, st);
  }
  // lmax 3, bf16: the same kernel, each slot in two channel halves (float32
  // rows of 8 KB would not fit two tiles of 16 in shared memory)
  if (s.lmax == 3 && bf && s.C == 128)
    return launch_eaas_tile<3, __nv_bfloat16>(s, d_x, pv.rec, items, d_w, d_y, st);
  switch (s.lmax) {
    case 1: return bf ? launch_eaas_t<1, __nv_bfloat16, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st)
                      : launch_eaas_t<1, float, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st);
    case 2: return bf ? launch_eaas_t<2, __nv_bfloat16, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st)
                      : launch_eaas_t<2, float, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st);
    case 3: return bf ? launch_eaas_t<3, __nv_bfloat16, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st)
                      : launch_eaas_t<3, float, true>(s, d_x, nullptr, pv.rec, items, d_w, d_y, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

int launch_eaas_planned_tf32out(const egat_shape& s, const void* d_x, const void* d_plan, const float* d_w,
                                float* d_y, cudaStream_t st) {
  if (s.dtype != EGAT_BF16 || s.C != 128) return EGAT_ERR_UNSUPPORTED;
  const PlanView pv = plan_view(const_cast<void*>(d_plan), s.n, s.K, s.lmax);
  const long long items = (long long)pv.tiles * kTileM;
  switch (s.lmax) {
    case 1: return launch_eaas_tile<1, __nv_bfloat16, Tf32Out>(s, d_x, pv.rec, items, d_w, d_y, st);
    case 2: return launch_eaas_tile<2, __nv_bfloat16, Tf32Out>(s, d_x, pv.rec, items, d_w, d_y, st);
    case 3: return launch_eaas_tile<3, __nv_bfloat16, Tf32Out>(s, d_x, pv.rec, items, d_w, d_y, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

int take_wait_timeouts_coupling(cudaStream_t st, unsigned int* count) {
  return take_unit_wait_timeouts(st, count) == 0 ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
