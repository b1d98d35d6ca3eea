// Device-side building blocks shared by the egat kernels: storage loads,
// compile-time coupling-path enumeration, real Wigner-D matrices and the
// per-channel EAAS operator.
//
// Pages cited (by title):
//  [EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构"
//  [TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation Memory"
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <type_traits>

namespace egat {

constexpr int kMaxL = 3;
constexpr int kMaxPaths = 34;
constexpr int kMaxDim = (kMaxL + 1) * (kMaxL + 1);

// ---------------------------------------------------------------------------
// compile-time helpers
// ---------------------------------------------------------------------------
template <int I, int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (I < N) {
    f(std::integral_constant<int, I>{});
    static_for<I + 1, N>(f);
  }
}

__host__ __device__ constexpr int iabs(int x) { return x < 0 ? -x : x; }

// Coupling paths (li, lf, lo): every triple <= L with |li-lf| <= lo <= li+lf,
// ordered by lo, then li, then lf ascending ([EX] §2.2 keeps both parities of
// li+lf+lo).  which: 0 -> li, 1 -> lf, 2 -> lo; p == -1 counts the paths.
__host__ __device__ constexpr int path_info(int L, int p, int which) {
  int n = 0;
  for (int lo = 0; lo <= L; ++lo)
    for (int li = 0; li <= L; ++li)
      for (int lf = 0; lf <= L; ++lf)
        if (iabs(li - lf) <= lo && lo <= li + lf) {
          if (n == p) return which == 0 ? li : (which == 1 ? lf : lo);
          ++n;
        }
  return p < 0 ? n : -1;
}
__host__ __device__ constexpr int num_paths(int L) { return path_info(L, -1, 0); }

// Offset of D^l inside the concatenated Wigner-D block (D^0, D^1, ...).
__host__ __device__ constexpr int wig_off(int l) {
  int o = 0;
  for (int k = 0; k < l; ++k) o += (2 * k + 1) * (2 * k + 1);
  return o;
}
__host__ __device__ constexpr int wig_size(int L) { return wig_off(L + 1); }

// Axis-frame re-index factors: for path p and output m_o, the factor that
// multiplies the rotated input component.  Filled on the host from
// Clebsch–Gordan coefficients; which input component it reads is fixed at
// compile time by the parity of li+lf+lo ([EX] §2.2; [TS] Eq. 13).
struct EaasTable {
  float f[kMaxPaths][2 * kMaxL + 1];
};

// Real-basis rotation generators of degrees 0..kMaxL for the three axes:
// J[a] holds, block-diagonally at wig_off(l), the (2l+1) x (2l+1) matrix
// dD^l(R_a(t))/dt at t = 0 (R_a(t) the rotation by t about axis a) of this
// library's own Wigner-D construction.  Filled on the host.
struct GenTable {
  float J[3][(kMaxL + 1) * (2 * kMaxL + 1) * (2 * kMaxL + 3) / 3];
};

// ---------------------------------------------------------------------------
// packed float2 arithmetic (sm_100 f32x2 FMA / MUL on a 64-bit register pair)
// ---------------------------------------------------------------------------
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// d = a * b + c, element-wise on (lo, hi)
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// two bf16 in one 32-bit word (element 2i in the low half) -> (lo, hi) floats
__device__ __forceinline__ f32x2 bf16x2_to_f2(uint32_t w) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xffff0000u));
  return r;
}

// ---------------------------------------------------------------------------
// storage loads / stores
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&o)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// 8 consecutive elements starting at an element offset that is a multiple of 8.
template <typename T>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    v = __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void to_f32(float (&o)[8]) const { bf16x8_to_f32(v, o); }
  // element pairs (0,1), (2,3), (4,5), (6,7) as packed floats
  __device__ __forceinline__ void to_f2(f32x2 (&o)[4]) const {
    o[0] = bf16x2_to_f2(v.x);
    o[1] = bf16x2_to_f2(v.y);
    o[2] = bf16x2_to_f2(v.z);
    o[3] = bf16x2_to_f2(v.w);
  }
};

template <>
struct Chunk8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void zero() {
    a = make_float4(0.f, 0.f, 0.f, 0.f);
    b = a;
  }
  __device__ __forceinline__ void to_f32(float (&o)[8]) const {
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  __device__ __forceinline__ void to_f2(f32x2 (&o)[4]) const {
    o[0] = f2_pack(a.x, a.y);
    o[1] = f2_pack(a.z, a.w);
    o[2] = f2_pack(b.x, b.y);
    o[3] = f2_pack(b.z, b.w);
  }
};

template <typename T>
__device__ __forceinline__ float load_one(const T* p);
template <>
__device__ __forceinline__ float load_one<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_one<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

template <typename T>
__device__ __forceinline__ void store_one(T* p, float v);
template <>
__device__ __forceinline__ void store_one<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_one<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// 2^x on the special-function unit (PTX ex2.approx).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// alignment rotation and real Wigner-D matrices
// ---------------------------------------------------------------------------
// Q = R_z(phi) R_y(theta), (theta, phi) the polar angles of r, so Q z = r/|r|
// ([EX] §2.1 "compute_alignment_rotation"); identity for r = 0.  Written with
// cos/sin of the angles taken directly from the coordinates.  Also returns
// |r|.  Row-major Q[3][3].
__device__ __forceinline__ float alignment_rotation(float x, float y, float z, float (&Q)[9]) {
  const float rho2 = x * x + y * y;
  const float r = sqrtf(rho2 + z * z);
  if (r == 0.f) {
    Q[0] = 1.f; Q[1] = 0.f; Q[2] = 0.f;
    Q[3] = 0.f; Q[4] = 1.f; Q[5] = 0.f;
    Q[6] = 0.f; Q[7] = 0.f; Q[8] = 1.f;
    return 0.f;
  }
  const float rho = sqrtf(rho2);
  const float ct = z / r, st = rho / r;
  float cp = 1.f, sp = 0.f;
  if (rho > 0.f) {
    cp = x / rho;
    sp = y / rho;
  }
  Q[0] = cp * ct; Q[1] = -sp; Q[2] = cp * st;
  Q[3] = sp * ct; Q[4] = cp;  Q[5] = sp * st;
  Q[6] = -st;     Q[7] = 0.f; Q[8] = ct;
  return r;
}

// Degree-1 real Wigner-D entry e = 3a + b: the rotation in (y, z, x) order.
__host__ __device__ constexpr int wig1_src(int e) {
  return ((e / 3 + 1) % 3) * 3 + ((e % 3 + 1) % 3);
}

// One entry D^l[m][mp] (m, mp in -l..l) of the real Wigner-D matrix of degree
// l >= 2, from D^1 and D^{l-1} by the recursion of Ivanic and Ruedenberg
// ("Rotation matrices for real spherical harmonics. Direct determination by
// recursion", J. Phys. Chem. 100 (1996) 6342; erratum 102 (1998) 9099).
// D1 and Dp are row-major with rows/cols indexed m + 1 and m + l - 1.
__device__ __forceinline__ float ir_entry(int l, int m, int mp, const float* D1,
                                          const float* Dp) {
  const int wp = 2 * l - 1;  // width of D^{l-1}
  auto r1 = [&](int i, int j) { return D1[(i + 1) * 3 + (j + 1)]; };
  auto rp = [&](int a, int b) { return Dp[(a + l - 1) * wp + (b + l - 1)]; };
  auto P = [&](int i, int a, int b) -> float {
    if (b == l) return r1(i, 1) * rp(a, l - 1) - r1(i, -1) * rp(a, -l + 1);
    if (b == -l) return r1(i, 1) * rp(a, -l + 1) + r1(i, -1) * rp(a, l - 1);
    return r1(i, 0) * rp(a, b);
  };
  const float d = (iabs(mp) == l) ? float((2 * l) * (2 * l - 1)) : float((l + mp) * (l - mp));
  const int am = iabs(m);
  const bool m0 = (m == 0);
  float val = 0.f;
  // u-term
  if (am < l) val += sqrtf(float((l + m) * (l - m)) / d) * P(0, m, mp);
  // v-term
  {
    const float v = 0.5f * sqrtf(float((m0 ? 2 : 1) * (l + am - 1) * (l + am)) / d) * (m0 ? -1.f : 1.f);
    float V;
    if (m0) {
      V = P(1, 1, mp) + P(-1, -1, mp);
    } else if (m > 0) {
      V = P(1, m - 1, mp) * (m == 1 ? 1.41421356237309515f : 1.f) -
          (m == 1 ? 0.f : P(-1, -m + 1, mp));
    } else {
      V = (m == -1 ? 0.f : P(1, m + 1, mp)) +
          P(-1, -m - 1, mp) * (m == -1 ? 1.41421356237309515f : 1.f);
    }
    val += v * V;
  }
  // w-term (vanishes for m = 0 and |m| >= l-1)
  if (!m0 && am < l - 1) {
    const float w = -0.5f * sqrtf(float((l - am - 1) * (l - am)) / d);
    const float W = (m > 0) ? (P(1, m + 1, mp) + P(-1, -m - 1, mp))
                            : (P(1, m - 1, mp) - P(-1, -m + 1, mp));
    val += w * W;
  }
  return val;
}

// The same recursion with every index and coefficient fixed at compile time:
// one thread builds all of D^0..D^L in registers, straight-line, with no
// branches, runtime square roots or shared memory.  D is the concatenated
// block (wig_off); D^1 and D^{l-1} are read from it while D^l is written.
__host__ __device__ constexpr double ct_sqrt(double x) {
  if (x <= 0.0) return 0.0;
  double r = x < 1.0 ? 1.0 : x;
  for (int i = 0; i < 200; ++i) r = 0.5 * (r + x / r);   // Newton; converged long before
  return r;
}
template <int l, int i, int a, int b, int N>
__device__ __forceinline__ float ir_P(const float (&D)[N]) {
  constexpr int o1 = wig_off(1), op = wig_off(l - 1), wp = 2 * l - 1;
  constexpr int row = op + (a + l - 1) * wp;
  if constexpr (b == l)
    return D[o1 + (i + 1) * 3 + 2] * D[row + 2 * l - 2] - D[o1 + (i + 1) * 3 + 0] * D[row];
  else if constexpr (b == -l)
    return D[o1 + (i + 1) * 3 + 2] * D[row] + D[o1 + (i + 1) * 3 + 0] * D[row + 2 * l - 2];
  else
    return D[o1 + (i + 1) * 3 + 1] * D[row + b + l - 1];
}
template <int l, int m, int mp, int N>
__device__ __forceinline__ float ir_entry_ct(const float (&D)[N]) {
  constexpr double d = (iabs(mp) == l) ? double((2 * l) * (2 * l - 1)) : double((l + mp) * (l - mp));
  constexpr int am = iabs(m);
  float val = 0.f;
  if constexpr (am < l) {
    constexpr float u = float(ct_sqrt(double((l + m) * (l - m)) / d));
    val += u * ir_P<l, 0, m, mp>(D);
  }
  {
    constexpr float v = float(0.5 * ct_sqrt(double((m == 0 ? 2 : 1) * (l + am - 1) * (l + am)) / d) *
                              (m == 0 ? -1.0 : 1.0));
    float V;
    if constexpr (m == 0) {
      V = ir_P<l, 1, 1, mp>(D) + ir_P<l, -1, -1, mp>(D);
    } else if constexpr (m == 1) {
      V = ir_P<l, 1, 0, mp>(D) * 1.41421356237309515f;
    } else if constexpr (m > 1) {
      V = ir_P<l, 1, m - 1, mp>(D) - ir_P<l, -1, -m + 1, mp>(D);
    } else if constexpr (m == -1) {
      V = ir_P<l, -1, 0, mp>(D) * 1.41421356237309515f;
    } else {
      V = ir_P<l, 1, m + 1, mp>(D) + ir_P<l, -1, -m - 1, mp>(D);
    }
    val += v * V;
  }
  if constexpr (m != 0 && am < l - 1) {
    constexpr float w = float(-0.5 * ct_sqrt(double((l - am - 1) * (l - am)) / d));
    float W;
    if constexpr (m > 0) W = ir_P<l, 1, m + 1, mp>(D) + ir_P<l, -1, -m - 1, mp>(D);
    else W = ir_P<l, 1, m - 1, mp>(D) - ir_P<l, -1, -m + 1, mp>(D);
    val += w * W;
  }
  return val;
}
template <int L>
__device__ __forceinline__ void wigner_regs(const float (&Q)[9], float (&D)[wig_size(L)]) {
  D[0] = 1.f;
  static_for<0, 9>([&](auto ec) {
    constexpr int e = decltype(ec)::value;
    D[wig_off(1) + e] = Q[wig1_src(e)];
  });
  static_for<2, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    static_for<0, w * w>([&](auto ec) {
      constexpr int e = decltype(ec)::value;
      D[wig_off(l) + e] = ir_entry_ct<l, e / w - l, e % w - l>(D);
    });
  });
}

// Build D^0..D^L for one rotation into Dsm (wig_size(L) floats) using
// `nthreads` cooperating threads (thread index `tid`); `sync` is called
// between degrees.  Dsm must be visible to all cooperating threads.
template <int L, typename Sync>
__device__ __forceinline__ void wigner_build(const float (&Q)[9], float* Dsm, int tid,
                                             int nthreads, Sync sync) {
  if (tid == 0) Dsm[0] = 1.f;
#pragma unroll
  for (int e = 0; e < 9; ++e)
    if (e % nthreads == tid) Dsm[wig_off(1) + e] = Q[wig1_src(e)];
  sync();
#pragma unroll
  for (int l = 2; l <= L; ++l) {
    const int w = 2 * l + 1;
    for (int e = tid; e < w * w; e += nthreads) {
      const int m = e / w - l, mp = e % w - l;
      Dsm[wig_off(l) + e] = ir_entry(l, m, mp, Dsm + wig_off(1), Dsm + wig_off(l - 1));
    }
    sync();
  }
}

// ---------------------------------------------------------------------------
// EAAS on one channel ([EX] §2.3, Proposition 4.3)
// ---------------------------------------------------------------------------
// y = sum_p w_p (x^{li} (x) R^{lf}(r))^{lo}, computed as
//   xt^l = D^l(Q)^T x^l                       (into the frame with z along r)
//   t^{lo}_m += w_p |r|^{lf} f_p(m) xt^{li}_{m or -m}   (only m_f = 0 survives)
//   y^l = D^l(Q) t^l                          (back to the global frame)
// `wgt(p)` returns w[p] for this channel; Dsm holds D^0..D^L.  x is
// overwritten (the rotation is done in place); each output component is
// handed to `out(d, value)` as soon as its degree is finished, so only x, t and
// one degree's worth of temporaries are live at a time.
template <int L, typename WFn, typename OutFn>
__device__ __forceinline__ void eaas_channel(float (&x)[(L + 1) * (L + 1)],
                                             const float* __restrict__ Dsm,
                                             const float (&rpow)[L + 1], const EaasTable& tab,
                                             WFn wgt, OutFn out) {
  constexpr int D = (L + 1) * (L + 1);
  float t[D];
#pragma unroll
  for (int i = 0; i < D; ++i) t[i] = 0.f;
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
    float tmp[w];
#pragma unroll
    for (int a = 0; a < w; ++a) {
      float s = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) s = fmaf(Dl[b * w + a], x[l * l + b], s);
      tmp[a] = s;
    }
#pragma unroll
    for (int a = 0; a < w; ++a) x[l * l + a] = tmp[a];
  });
  static_for<0, num_paths(L)>([&](auto pc) {
    constexpr int p = decltype(pc)::value;
    constexpr int li = path_info(L, p, 0);
    constexpr int lf = path_info(L, p, 1);
    constexpr int lo = path_info(L, p, 2);
    constexpr bool even = ((li + lf + lo) % 2) == 0;
    const float wp = wgt(p) * rpow[lf];
#pragma unroll
    for (int mo = -lo; mo <= lo; ++mo) {
      const int src = even ? mo : -mo;
      const bool live = (iabs(mo) <= li) && (even || mo != 0);
      if (live) t[lo * lo + lo + mo] = fmaf(wp * tab.f[p][mo + lo], x[li * li + li + src],
                                            t[lo * lo + lo + mo]);
    }
  });
  out(0, t[0]);
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
#pragma unroll
    for (int a = 0; a < w; ++a) {
      float s = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) s = fmaf(Dl[a * w + b], t[l * l + b], s);
      out(l * l + a, s);
    }
  });
}

// The transpose of eaas_channel for fixed r and weights (the adjoint used by
// the backward pass): the coupling is y = D Rw D^T x with Rw the weighted
// axis-frame re-index, so its transpose is D Rw^T D^T g — the same rotations
// around the re-index read backwards (output degree lo -> input degree li).
// g is overwritten; out(d, v) receives component d of the result.
template <int L, typename WFn, typename OutFn>
__device__ __forceinline__ void eaas_channel_adjoint(float (&g)[(L + 1) * (L + 1)],
                                                     const float* __restrict__ Dsm,
                                                     const float (&rpow)[L + 1],
                                                     const EaasTable& tab, WFn wgt, OutFn out) {
  constexpr int D = (L + 1) * (L + 1);
  float t[D];
#pragma unroll
  for (int i = 0; i < D; ++i) t[i] = 0.f;
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
    float tmp[w];
#pragma unroll
    for (int a = 0; a < w; ++a) {
      float s = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) s = fmaf(Dl[b * w + a], g[l * l + b], s);
      tmp[a] = s;
    }
#pragma unroll
    for (int a = 0; a < w; ++a) g[l * l + a] = tmp[a];
  });
  static_for<0, num_paths(L)>([&](auto pc) {
    constexpr int p = decltype(pc)::value;
    constexpr int li = path_info(L, p, 0);
    constexpr int lf = path_info(L, p, 1);
    constexpr int lo = path_info(L, p, 2);
    constexpr bool even = ((li + lf + lo) % 2) == 0;
    const float wp = wgt(p) * rpow[lf];
#pragma unroll
    for (int mo = -lo; mo <= lo; ++mo) {
      const int src = even ? mo : -mo;
      const bool live = (iabs(mo) <= li) && (even || mo != 0);
      if (live) t[li * li + li + src] = fmaf(wp * tab.f[p][mo + lo], g[lo * lo + lo + mo],
                                             t[li * li + li + src]);
    }
  });
  out(0, t[0]);
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
#pragma unroll
    for (int a = 0; a < w; ++a) {
      float s = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) s = fmaf(Dl[a * w + b], t[l * l + b], s);
      out(l * l + a, s);
    }
  });
}

// Position gradient of one channel's coupling value L_c = <g, T(x; r)> (T the
// operator of eaas_channel: T = D Rw D^T with D = D(Q), Q z = r/|r|, and Rw the
// weighted axis-frame re-index), evaluated in the aligned frame:
//   g~ = D^T g, x~ = D^T x;
//   dL_c/d|r| = <g~, Rw' x~>, Rw' with |r|^l replaced by l |r|^(l-1) (drpow);
//   rotating g, x and r together leaves L_c unchanged, so
//   r x grad L_c = -tau with tau_a = <J_a g, T x> + <g, T(J_a x)>, and since
//   D^T J_a D = sum_b Q_ab J_b, tau = Q tau~ with
//   tau~_b = <J_b g~, Rw x~> + <g~, Rw J_b x~>.
// With r = |r| Q z only tau~_x and tau~_y matter:
//   grad L_c = Q ( -tau~_y / |r|, tau~_x / |r|, dL_c/d|r| ).
// This accumulates dr, tx = tau~_x, ty = tau~_y for the caller.
template <int L, typename WFn>
__device__ __forceinline__ void coupling_grad_channel(float (&g)[(L + 1) * (L + 1)],
                                                      float (&x)[(L + 1) * (L + 1)],
                                                      const float* __restrict__ Dsm,
                                                      const float (&rpow)[L + 1],
                                                      const float (&drpow)[L + 1],
                                                      const EaasTable& tab, const GenTable& gen,
                                                      WFn wgt, float& dr, float& tx, float& ty) {
  constexpr int D = (L + 1) * (L + 1);
  // into the aligned frame (in place)
  auto to_frame = [&](float (&v)[D]) {
    static_for<1, L + 1>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      constexpr int w = 2 * l + 1;
      const float* Dl = Dsm + wig_off(l);
      float tmp[w];
#pragma unroll
      for (int a = 0; a < w; ++a) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < w; ++c) s = fmaf(Dl[c * w + a], v[l * l + c], s);
        tmp[a] = s;
      }
#pragma unroll
      for (int a = 0; a < w; ++a) v[l * l + a] = tmp[a];
    });
  };
  // <u, Rw(pw) v> for the re-index with radial factors pw
  auto reindex_dot = [&](const float (&u)[D], const float (&v)[D], const float (&pw)[L + 1]) {
    float acc = 0.f;
    static_for<0, num_paths(L)>([&](auto pc) {
      constexpr int p = decltype(pc)::value;
      constexpr int li = path_info(L, p, 0);
      constexpr int lf = path_info(L, p, 1);
      constexpr int lo = path_info(L, p, 2);
      constexpr bool even = ((li + lf + lo) % 2) == 0;
      const float wp = wgt(p) * pw[lf];
      float part = 0.f;
#pragma unroll
      for (int mo = -lo; mo <= lo; ++mo) {
        const int src = even ? mo : -mo;
        const bool live = (iabs(mo) <= li) && (even || mo != 0);
        if (live) part = fmaf(tab.f[p][mo + lo] * u[lo * lo + lo + mo], v[li * li + li + src], part);
      }
      acc = fmaf(wp, part, acc);
    });
    return acc;
  };
  // o = J_b v (block-diagonal)
  auto gen_apply = [&](int bax, const float (&v)[D], float (&o)[D]) {
    o[0] = 0.f;
    static_for<1, L + 1>([&](auto lc) {
      constexpr int l = decltype(lc)::value;
      constexpr int w = 2 * l + 1;
      const float* Jl = gen.J[bax] + wig_off(l);
#pragma unroll
      for (int m = 0; m < w; ++m) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < w; ++c) s = fmaf(Jl[m * w + c], v[l * l + c], s);
        o[l * l + m] = s;
      }
    });
  };
  to_frame(g);
  to_frame(x);
  if constexpr (L >= 3) {
    // One pass over the paths with all five dot products at once, so that
    // each path's weight and factors are read for one use: at lmax 3 the
    // five separate passes keep them live across passes, past the registers.
    float jgx[D], jxx[D], jgy[D], jxy[D];
    gen_apply(0, g, jgx);
    gen_apply(0, x, jxx);
    gen_apply(1, g, jgy);
    gen_apply(1, x, jxy);
    float adr = 0.f, atx = 0.f, aty = 0.f;
    static_for<0, num_paths(L)>([&](auto pc) {
      constexpr int p = decltype(pc)::value;
      constexpr int li = path_info(L, p, 0);
      constexpr int lf = path_info(L, p, 1);
      constexpr int lo = path_info(L, p, 2);
      constexpr bool even = ((li + lf + lo) % 2) == 0;
      const float w = wgt(p);
      float pdr = 0.f, ptx = 0.f, pty = 0.f;
#pragma unroll
      for (int mo = -lo; mo <= lo; ++mo) {
        const int src = even ? mo : -mo;
        const bool live = (iabs(mo) <= li) && (even || mo != 0);
        if (live) {
          const int uo = lo * lo + lo + mo, vi = li * li + li + src;
          const float f = tab.f[p][mo + lo];
          pdr = fmaf(f * g[uo], x[vi], pdr);
          ptx = fmaf(f, fmaf(jgx[uo], x[vi], g[uo] * jxx[vi]), ptx);
          pty = fmaf(f, fmaf(jgy[uo], x[vi], g[uo] * jxy[vi]), pty);
        }
      }
      adr = fmaf(w * drpow[lf], pdr, adr);
      atx = fmaf(w * rpow[lf], ptx, atx);
      aty = fmaf(w * rpow[lf], pty, aty);
    });
    dr += adr;
    tx += atx;
    ty += aty;
    return;
  }
  dr += reindex_dot(g, x, drpow);
  // <J_b g~, Rw x~> = <Rw^T J_b g~, x~> = reindex_dot(J_b g~, x~); <g~, Rw J_b x~> = reindex_dot(g~, J_b x~)
#pragma unroll 1
  for (int bax = 0; bax < 2; ++bax) {
    float jv[D];
    gen_apply(bax, g, jv);
    float s = reindex_dot(jv, x, rpow);
    gen_apply(bax, x, jv);
    s += reindex_dot(g, jv, rpow);
    tx += bax == 0 ? s : 0.f;
    ty += bax == 1 ? s : 0.f;
  }
}

// eaas_multi on channel pairs: the same operations in the same order per
// channel, each pair of channels in one packed f32x2 FMA (or MUL), so the
// results equal the scalar form bit for bit with about half the FP
// instructions.
template <int L, int NP, typename WFn, typename OutFn>
__device__ __forceinline__ void eaas_multi_packed(float (&x)[2 * NP][(L + 1) * (L + 1)],
                                                  const float* __restrict__ Dsm,
                                                  const float (&rpow)[L + 1], const EaasTable& tab,
                                                  WFn wgt, OutFn out) {
  constexpr int D = (L + 1) * (L + 1);
  f32x2 xv[NP][D], t[NP][D];
#pragma unroll
  for (int j = 0; j < NP; ++j)
#pragma unroll
    for (int d = 0; d < D; ++d) {
      xv[j][d] = f2_pack(x[2 * j][d], x[2 * j + 1][d]);
      t[j][d] = 0ull;   // (+0, +0)
    }
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
    f32x2 tmp[NP][w];
#pragma unroll
    for (int a = 0; a < w; ++a) {
#pragma unroll
      for (int j = 0; j < NP; ++j) tmp[j][a] = 0ull;
#pragma unroll
      for (int b = 0; b < w; ++b) {
        const float dv = Dl[b * w + a];
        const f32x2 d2 = f2_pack(dv, dv);
#pragma unroll
        for (int j = 0; j < NP; ++j) tmp[j][a] = f2_fma(d2, xv[j][l * l + b], tmp[j][a]);
      }
    }
#pragma unroll
    for (int j = 0; j < NP; ++j)
#pragma unroll
      for (int a = 0; a < w; ++a) xv[j][l * l + a] = tmp[j][a];
  });
  static_for<0, num_paths(L)>([&](auto pc) {
    constexpr int p = decltype(pc)::value;
    constexpr int li = path_info(L, p, 0);
    constexpr int lf = path_info(L, p, 1);
    constexpr int lo = path_info(L, p, 2);
    constexpr bool even = ((li + lf + lo) % 2) == 0;
    f32x2 wp[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) wp[j] = f2_pack(wgt(p, 2 * j) * rpow[lf], wgt(p, 2 * j + 1) * rpow[lf]);
#pragma unroll
    for (int mo = -lo; mo <= lo; ++mo) {
      const int src = even ? mo : -mo;
      const bool live = (iabs(mo) <= li) && (even || mo != 0);
      if (live) {
        const float f = tab.f[p][mo + lo];
        const f32x2 f2 = f2_pack(f, f);
#pragma unroll
        for (int j = 0; j < NP; ++j)
          t[j][lo * lo + lo + mo] = f2_fma(f2_mul(wp[j], f2), xv[j][li * li + li + src], t[j][lo * lo + lo + mo]);
      }
    }
  });
  {
    float y[2 * NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) f2_unpack(t[j][0], y[2 * j], y[2 * j + 1]);
    out(0, y);
  }
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
#pragma unroll
    for (int a = 0; a < w; ++a) {
      f32x2 y2[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) y2[j] = 0ull;
#pragma unroll
      for (int b = 0; b < w; ++b) {
        const float dv = Dl[a * w + b];
        const f32x2 d2 = f2_pack(dv, dv);
#pragma unroll
        for (int j = 0; j < NP; ++j) y2[j] = f2_fma(d2, t[j][l * l + b], y2[j]);
      }
      float y[2 * NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) f2_unpack(y2[j], y[2 * j], y[2 * j + 1]);
      out(l * l + a, y);
    }
  });
}

// The same operator on NCH channels at once (channels of one atom share the
// Wigner-D matrices): each matrix entry is read once and applied to every
// channel.  x[k][d] is overwritten; wgt(p, k) returns w[p] of channel k;
// out(d, y) receives component d of all NCH channels.  PACKED (an even NCH)
// runs the channels as packed pairs, for callers with registers to spare.
template <int L, int NCH, bool PACKED = false, typename WFn, typename OutFn>
__device__ __forceinline__ void eaas_multi(float (&x)[NCH][(L + 1) * (L + 1)],
                                           const float* __restrict__ Dsm,
                                           const float (&rpow)[L + 1], const EaasTable& tab,
                                           WFn wgt, OutFn out) {
  if constexpr (PACKED) {
    static_assert(NCH % 2 == 0, "channel pairs");
    eaas_multi_packed<L, NCH / 2>(x, Dsm, rpow, tab, wgt, out);
  } else {
  constexpr int D = (L + 1) * (L + 1);
  float t[NCH][D];
#pragma unroll
  for (int k = 0; k < NCH; ++k)
#pragma unroll
    for (int i = 0; i < D; ++i) t[k][i] = 0.f;
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
    float tmp[NCH][w];
#pragma unroll
    for (int a = 0; a < w; ++a) {
#pragma unroll
      for (int k = 0; k < NCH; ++k) tmp[k][a] = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) {
        const float dv = Dl[b * w + a];
#pragma unroll
        for (int k = 0; k < NCH; ++k) tmp[k][a] = fmaf(dv, x[k][l * l + b], tmp[k][a]);
      }
    }
#pragma unroll
    for (int k = 0; k < NCH; ++k)
#pragma unroll
      for (int a = 0; a < w; ++a) x[k][l * l + a] = tmp[k][a];
  });
  static_for<0, num_paths(L)>([&](auto pc) {
    constexpr int p = decltype(pc)::value;
    constexpr int li = path_info(L, p, 0);
    constexpr int lf = path_info(L, p, 1);
    constexpr int lo = path_info(L, p, 2);
    constexpr bool even = ((li + lf + lo) % 2) == 0;
    float wp[NCH];
#pragma unroll
    for (int k = 0; k < NCH; ++k) wp[k] = wgt(p, k) * rpow[lf];
#pragma unroll
    for (int mo = -lo; mo <= lo; ++mo) {
      const int src = even ? mo : -mo;
      const bool live = (iabs(mo) <= li) && (even || mo != 0);
      if (live) {
        const float f = tab.f[p][mo + lo];
#pragma unroll
        for (int k = 0; k < NCH; ++k)
          t[k][lo * lo + lo + mo] = fmaf(wp[k] * f, x[k][li * li + li + src], t[k][lo * lo + lo + mo]);
      }
    }
  });
  {
    float y[NCH];
#pragma unroll
    for (int k = 0; k < NCH; ++k) y[k] = t[k][0];
    out(0, y);
  }
  static_for<1, L + 1>([&](auto lc) {
    constexpr int l = decltype(lc)::value;
    constexpr int w = 2 * l + 1;
    const float* Dl = Dsm + wig_off(l);
#pragma unroll
    for (int a = 0; a < w; ++a) {
      float y[NCH];
#pragma unroll
      for (int k = 0; k < NCH; ++k) y[k] = 0.f;
#pragma unroll
      for (int b = 0; b < w; ++b) {
        const float dv = Dl[a * w + b];
#pragma unroll
        for (int k = 0; k < NCH; ++k) y[k] = fmaf(dv, t[k][l * l + b], y[k]);
      }
      out(l * l + a, y);
    }
  });
  }
}

}  // namespace egat
