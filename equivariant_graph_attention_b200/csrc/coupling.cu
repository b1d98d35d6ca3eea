// Step 2: EAAS source coupling h'_j = h_j (x) R(r_j).
//
// [EX] = "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §2.1-§2.3
// (alignment rotation, sparse re-index, Proposition 4.3), §3.1 step 1;
// [TS] = "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
// Memory" §2.1 (Lemma 4.1: only m = 0 of the solid harmonic survives in the
// aligned frame; Eq. 13: the re-index rule).
//
// Kernel layout: one thread per (atom, channel); a warp covers 32 channels of
// one atom (or all 16 channels of two atoms).  The warp builds the atom's
// Wigner-D matrices (degree 1 from the alignment rotation, higher degrees by
// the Ivanic–Ruedenberg recursion, entries in parallel) in shared memory;
// each lane then rotates its channel's components into the aligned frame,
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
  EaasTable tab;
};

// One warp owns a block of G = min(C, 32) channels of 32/G atoms at a time
// (lane = channel, so every load and store of a component row is coalesced).
// The warp's channel block is fixed, so the path weights of its lane's channel
// stay in registers.  Each warp builds the Wigner-D matrices of its atoms in
// its own shared-memory slot with warp-level synchronisation only, and the
// next atom's position and features are fetched before the current atom is
// coupled.
template <int L, typename T>
__global__ void __launch_bounds__(kEaasWarps * 32, (L >= 3 ? 1 : 2))
eaas_source_kernel(const __grid_constant__ EaasParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int NP = num_paths(L);
  constexpr int WS = wig_size(L);
  __shared__ float Dsm[kEaasWarps][2][WS];   // up to 2 atoms per warp (C = 16)

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int C = p.C;
  const int G = C < 32 ? C : 32;          // lanes per atom
  const int AW = 32 / G;                  // atoms per warp (1 or 2)
  const int slot = lane / G;              // which of the warp's atoms
  const int g = lane % G;
  const int nblk = C / G;                 // channel blocks per atom
  const long long gwarp = (long long)blockIdx.x * kEaasWarps + wib;
  const long long nwarps = (long long)gridDim.x * kEaasWarps;
  const int cb = int(gwarp % nblk);
  const int c = cb * G + g;               // this lane's channel
  const long long ngroups = ((long long)p.n + AW - 1) / AW;
  const T* __restrict__ x = static_cast<const T*>(p.x);
  T* __restrict__ y = static_cast<T*>(p.y);

  // weights of this lane's channel: registers up to lmax 2, L1-cached loads above
  constexpr bool kRegW = NP <= 15;
  float wreg[kRegW ? NP : 1];
#pragma unroll
  for (int q = 0; q < (kRegW ? NP : 0); ++q) wreg[q] = __ldg(p.w + q * C + c);
  const float* __restrict__ wcol = p.w + c;

  float* Dme = Dsm[wib][slot];
  long long grp = gwarp / nblk;
  const long long gstride = nwarps / nblk;   // launch keeps nwarps a multiple of nblk

  // prefetch the first atom
  float px = 0.f, py = 0.f, pz = 0.f, xin[D];
  auto fetch = [&](long long gr, float& fx, float& fy, float& fz, float (&xv)[D]) {
    const long long at = gr * AW + slot;
    if (gr < ngroups && at < p.n) {
      fx = __ldg(p.pos + 3 * at);
      fy = __ldg(p.pos + 3 * at + 1);
      fz = __ldg(p.pos + 3 * at + 2);
      const T* xr = x + (size_t)at * D * C + c;
#pragma unroll
      for (int d = 0; d < D; ++d) xv[d] = load_one<T>(xr + d * C);
    }
  };
  fetch(grp, px, py, pz, xin);
  // lmax 3 keeps no second feature row in flight (register budget)
  constexpr bool kPrefetch = L <= 2;
  for (; grp < ngroups; grp += gstride) {
    const long long at = grp * AW + slot;
    float nx = 0.f, ny = 0.f, nz = 0.f, xnext[kPrefetch ? D : 1];
    if constexpr (kPrefetch) fetch(grp + gstride, nx, ny, nz, xnext);
    float Q[9];
    const float r = alignment_rotation(px, py, pz, Q);
    float rpow[L + 1];
    rpow[0] = 1.f;
#pragma unroll
    for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
    __syncwarp();                             // previous atom's readers are done
    wigner_build<L>(Q, Dme, g, G, [] { __syncwarp(); });
    if (at < p.n) {
      T* yr = y + (size_t)at * D * C + c;
      eaas_channel<L>(
          xin, Dme, rpow, p.tab,
          [&](int q) {
            if constexpr (kRegW) return wreg[q];
            else return __ldg(wcol + q * C);
          },
          [&](int d, float v) { store_one<T>(yr + d * C, v); });
    }
    if constexpr (kPrefetch) {
      px = nx;
      py = ny;
      pz = nz;
#pragma unroll
      for (int d = 0; d < D; ++d) xin[d] = xnext[d];
    } else {
      fetch(grp + gstride, px, py, pz, xin);
    }
  }
}

template <int L, typename T>
int launch_eaas_t(const egat_shape& s, const void* d_x, const float* d_pos, const float* d_w,
                  void* d_y, cudaStream_t st) {
  EaasParams p;
  p.x = d_x;
  p.pos = d_pos;
  p.w = d_w;
  p.y = d_y;
  p.n = s.n;
  p.C = s.C;
  p.tab = eaas_table(L);
  const int G = s.C < 32 ? s.C : 32;
  const int nblk = s.C / G;
  const long long groups = ((long long)s.n + (32 / G) - 1) / (32 / G);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // warps needed: one per (atom group, channel block); cap at 8 resident blocks per SM
  const long long want = (groups * nblk + kEaasWarps - 1) / kEaasWarps;
  int grid = int(std::max<long long>(1, std::min<long long>(want, (long long)sms * 8)));
  // keep the total warp count a multiple of the channel-block count
  while ((long long)grid * kEaasWarps % nblk) ++grid;
  eaas_source_kernel<L, T><<<grid, kEaasWarps * 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace

int launch_eaas_source(const egat_shape& s, const void* d_x, const float* d_pos,
                       const float* d_w, void* d_y, cudaStream_t st) {
  const bool bf = s.dtype == EGAT_BF16;
  switch (s.lmax) {
    case 1: return bf ? launch_eaas_t<1, __nv_bfloat16>(s, d_x, d_pos, d_w, d_y, st)
                      : launch_eaas_t<1, float>(s, d_x, d_pos, d_w, d_y, st);
    case 2: return bf ? launch_eaas_t<2, __nv_bfloat16>(s, d_x, d_pos, d_w, d_y, st)
                      : launch_eaas_t<2, float>(s, d_x, d_pos, d_w, d_y, st);
    case 3: return bf ? launch_eaas_t<3, __nv_bfloat16>(s, d_x, d_pos, d_w, d_y, st)
                      : launch_eaas_t<3, float>(s, d_x, d_pos, d_w, d_y, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

}  // namespace egat
