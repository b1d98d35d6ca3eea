// Step 2: EAAS source coupling h'_j = h_j (x) R(r_j).
//
// [EX] = "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §2.1-§2.3
// (alignment rotation, sparse re-index, Proposition 4.3), §3.1 step 1;
// [TS] = "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
// Memory" §2.1 (Lemma 4.1: only m = 0 of the solid harmonic survives in the
// aligned frame; Eq. 13: the re-index rule).
//
// Kernel layout: a 256-thread block takes tiles of 256/C atoms, one thread per
// (atom, channel).  Per tile the block builds each atom's Wigner-D matrices
// (degree 1 from the alignment rotation, higher degrees by the
// Ivanic–Ruedenberg recursion, entries in parallel) in shared memory; each
// thread then rotates its channel's components into the aligned frame,
// applies the sparse re-index with the path weights, and rotates back.  The
// weights of the thread's channel stay in registers across tiles.  Memory
// traffic is one read of h and one write of h' (streaming, HBM-bound).
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

constexpr int kEaasThreads = 256;

struct EaasParams {
  const void* x;
  const float* pos;
  const float* w;
  void* y;
  int n;
  int C;
  EaasTable tab;
};

template <int L, typename T>
__global__ void __launch_bounds__(kEaasThreads)
eaas_source_kernel(const __grid_constant__ EaasParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int NP = num_paths(L);
  constexpr int WS = wig_size(L);
  constexpr int kMaxAtoms = kEaasThreads / 16;
  __shared__ float Dsm[kMaxAtoms][WS];
  __shared__ float Qs[kMaxAtoms][9];
  __shared__ float rps[kMaxAtoms][L + 1];

  const int C = p.C;
  const int A = kEaasThreads / C;  // atoms per tile
  const int tid = threadIdx.x;
  const int a = tid / C;           // atom slot of this thread
  const int c = tid % C;           // channel of this thread
  const T* __restrict__ x = static_cast<const T*>(p.x);
  T* __restrict__ y = static_cast<T*>(p.y);

  float wreg[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) wreg[q] = __ldg(p.w + q * C + c);

  const int ntiles = (p.n + A - 1) / A;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int atom0 = tile * A;
    if (tid < A) {
      const int at = atom0 + tid;
      float Q[9];
      float r = 0.f;
      if (at < p.n) {
        r = alignment_rotation(p.pos[3 * at], p.pos[3 * at + 1], p.pos[3 * at + 2], Q);
      } else {
        alignment_rotation(0.f, 0.f, 0.f, Q);
      }
#pragma unroll
      for (int e = 0; e < 9; ++e) Qs[tid][e] = Q[e];
      float rp = 1.f;
#pragma unroll
      for (int l = 0; l <= L; ++l) {
        rps[tid][l] = rp;
        rp *= r;
      }
    }
    __syncthreads();
    {
      float Q[9];
#pragma unroll
      for (int e = 0; e < 9; ++e) Q[e] = Qs[a][e];
      wigner_build<L>(Q, Dsm[a], c, C, [] { __syncthreads(); });
    }
    const int at = atom0 + a;
    if (at < p.n) {
      float xin[D], yout[D], rpow[L + 1];
#pragma unroll
      for (int l = 0; l <= L; ++l) rpow[l] = rps[a][l];
      const T* xr = x + (size_t)at * D * C + c;
#pragma unroll
      for (int d = 0; d < D; ++d) xin[d] = load_one<T>(xr + d * C);
      eaas_channel<L>(xin, yout, Dsm[a], rpow, p.tab, [&](int q) { return wreg[q]; });
      T* yr = y + (size_t)at * D * C + c;
#pragma unroll
      for (int d = 0; d < D; ++d) store_one<T>(yr + d * C, yout[d]);
    }
    __syncthreads();
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
  const int A = kEaasThreads / s.C;
  const int ntiles = (s.n + A - 1) / A;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(ntiles, sms * 8));
  eaas_source_kernel<L, T><<<grid, kEaasThreads, 0, st>>>(p);
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
