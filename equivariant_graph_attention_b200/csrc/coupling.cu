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
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
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
  static __device__ __forceinline__ void store(float* p, const float (&v)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
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
template <int L, typename T, bool PLANNED>
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
  constexpr int REC = kTileM * (1 + (L + 1) + WS);
  const T* __restrict__ x = static_cast<const T*>(p.x);
  T* __restrict__ y = static_cast<T*>(p.y);
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
        at = reinterpret_cast<const int*>(R)[rs];
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
      for (int l = 0; l <= L; ++l) rpow[l] = live ? __ldg(R + kTileM + rs * (L + 1) + l) : 0.f;
      __syncwarp();                           // previous atom's readers are done
      if (live)
        for (int e = gl; e < WS; e += GW) Dme[e] = __ldg(R + kTileM * (2 + L) + rs * WS + e);
      __syncwarp();
    } else {
      rpow[0] = 1.f;
#pragma unroll
      for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
      __syncwarp();                           // previous atom's readers are done
      wigner_build<L>(Q, Dme, gl, GW, [] { __syncwarp(); });
    }
    if (live) {
      T* yr = y + (size_t)at * D * C + c0;
      const float* swc = sw + c0;
      eaas_multi<L, CPL>(xv, Dme, rpow, p.tab, [&](int q, int k) { return swc[q * C + k]; },
                         [&](int d, const float (&v)[CPL]) { ChanVec<T, CPL>::store(yr + d * C, v); });
    }
  }
}
template <int L, typename T, bool PLANNED>
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
  eaas_source_kernel<L, T, PLANNED><<<grid, kEaasWarps * 32, shmem, st>>>(p);
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

int launch_eaas_planned(const egat_shape& s, const void* d_x, const void* d_plan, const float* d_w,
                        void* d_y, cudaStream_t st) {
  const bool bf = s.dtype == EGAT_BF16;
  const PlanView pv = plan_view(const_cast<void*>(d_plan), s.n, s.K, s.lmax);
  const long long items = (long long)pv.tiles * kTileM;
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

}  // namespace egat
