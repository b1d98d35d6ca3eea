// Backward pass of steps 2-4: the gradients of L = sum_i <G_i, ^h_i> with
// respect to the features h, the queries q and the keys k, for an upstream
// gradient G = dL/d^h.
//
// The pages name the backward pass as the step after the forward (forces as
// energy gradients in the Conservative mode) and keep the attention weights
// off HBM ("E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.2, linear
// activation memory; "E2Former-V2: On-the-Fly Equivariant Attention with
// Linear Activation Memory" §2.2).  Here too no per-edge quantity is stored:
// every weight is recomputed from q, k and one log-sum-exp per (target,
// head).  Steps, each the adjoint of a forward step:
//  1. dm = T*(G; r, w2): the target coupling is linear in m, so its adjoint
//     is the same rotate / re-index / rotate-back operator with the re-index
//     read backwards (eaas_channel_adjoint).  h' and dm are held in float32
//     whatever the storage type: the softmax backward subtracts nearly equal
//     quantities (dalpha - Delta), and bf16 intermediates there cost up to 3e-2
//     relative error on single (atom, head) rows of dq and dk;
//  2. the neighbour lists are transposed (in-lists: the targets each atom
//     serves), sorted so every sum runs in a fixed order;
//  3. per target i (one warp): a sweep over the key rows gives the per-head
//     log-sum-exp; one sweep over key and value rows then gives the exact
//     weights alpha_ij, m_i, Delta_i = sum_j alpha_ij dalpha_ij per head
//     (dalpha_ij = <dm_i, h'_j>_head) and dq_i = sum_j ds_ij k_j / sqrt(dk) with
//     ds_ij = alpha_ij (dalpha_ij - Delta_i), accumulated as
//     sum alpha dalpha k - Delta sum alpha k;
//  4. per source j (one warp) over its in-list: alpha_ij from q_i, k_j and
//     the target's log-sum-exp, dh'_j = sum_i alpha_ij dm_i,
//     dk_j = sum_i ds_ij q_i / sqrt(dk); the epilogue applies the adjoint of
//     the source coupling, dh_j = T*(dh'_j; r_j, w1).
// Step 2's in-lists make every gradient a gather: no atomics touch a result.
//  5. (optional) dL/dr: positions enter only through the solid harmonics of
//     the two couplings.  For each coupling value <g, T(x; r)> the radial
//     derivative is the same operator with |r|^l -> l |r|^(l-1), and the
//     angular part follows from equivariance: rotating g, x and r together
//     leaves it unchanged, so r x grad = -(<J g, T x> + <g, T(J x)>) with J the
//     rotation generators of the Wigner-D representation; both are evaluated
//     in the frame aligned with r (coupling_grad_channel).
//     The target pass adds the target coupling's part (g = G_i, x = m_i), the
//     source pass the source coupling's (g = dh'_j, x = h_j).
#include <cfloat>
#include <climits>
#include <cmath>
#include <mutex>

#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kBwdWarps = 4;   // (3 CTAs per SM for the attention passes: no spills at 168 registers)
constexpr int kSortCap = 4096;   // in-list length sorted in shared memory

// ---------------------------------------------------------------- step 1
// float -> the nearest tf32 value (ties away), as a float
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// TF32: the result rounded to tf32 (the tiled passes' operand format)
template <int L, typename T, bool TF32 = false>
__global__ void __launch_bounds__(kBwdWarps * 32)
adjoint_coupling_kernel(const float* __restrict__ g, const float* __restrict__ pos,
                        const float* __restrict__ w, T* __restrict__ out, int n, int C,
                        const __grid_constant__ EaasTable tab) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int WS = wig_size(L);
  __shared__ float Dsm[kBwdWarps][WS];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int a = blockIdx.x * kBwdWarps + wib;
  if (a >= n) return;   // whole warp
  float Q[9];
  const float r = alignment_rotation(pos[3 * a], pos[3 * a + 1], pos[3 * a + 2], Q);
  float rpow[L + 1];
  rpow[0] = 1.f;
#pragma unroll
  for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
  wigner_build<L>(Q, Dsm[wib], lane, 32, [] { __syncwarp(); });
  __syncwarp();
  for (int c = lane; c < C; c += 32) {
    float x[D];
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = g[((size_t)a * D + d) * C + c];
    eaas_channel_adjoint<L>(x, Dsm[wib], rpow, tab, [&](int pp) { return __ldg(w + pp * C + c); },
                            [&](int d, float v) {
                              store_one<T>(out + ((size_t)a * D + d) * C + c, TF32 ? round_tf32(v) : v);
                            });
  }
}

// The same operator with each atom's rotation and |r|^l taken from the
// attention plan's tile records instead of built per atom: one warp per tile
// slot copies the slot's Wigner-D into its shared memory.
template <int L, typename T, bool TF32 = false>
__global__ void __launch_bounds__(kBwdWarps * 32)
adjoint_planned_kernel(const float* __restrict__ g, const float* __restrict__ rec, long long items,
                       const float* __restrict__ w, T* __restrict__ out, int n, int C,
                       const __grid_constant__ EaasTable tab) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int WS = wig_size(L);
  constexpr int REC = plan_record_words(L);
  static_assert(WS == rec_wig_size(L), "record and shared-memory Wigner-D layouts agree");
  __shared__ float Dsm[kBwdWarps][WS];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long long slot = (long long)blockIdx.x * kBwdWarps + wib;
  if (slot >= items) return;   // whole warp
  const float* rc = rec + (slot / kTileM) * REC;
  const int r = int(slot % kTileM);
  const int a = reinterpret_cast<const int*>(rc)[kRecTgt + r];
  if ((unsigned)a >= (unsigned)n) return;   // an empty slot of the last tile
  for (int e = lane; e < WS; e += 32) Dsm[wib][e] = __ldg(rc + rec_off_D(L) + r * WS + e);
  float rpow[L + 1];
#pragma unroll
  for (int l = 0; l <= L; ++l) rpow[l] = __ldg(rc + kRecRp + r * (L + 1) + l);
  __syncwarp();
  for (int c = lane; c < C; c += 32) {
    float x[D];
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = g[((size_t)a * D + d) * C + c];
    eaas_channel_adjoint<L>(x, Dsm[wib], rpow, tab, [&](int pp) { return __ldg(w + pp * C + c); },
                            [&](int d, float v) {
                              store_one<T>(out + ((size_t)a * D + d) * C + c, TF32 ? round_tf32(v) : v);
                            });
  }
}

// ---------------------------------------------------------------- step 2
__device__ __forceinline__ int row_count(const int32_t* cnt, int i, int K) {
  int c = cnt ? cnt[i] : K;
  return c < 0 ? 0 : (c > K ? K : c);
}

__global__ void in_degree_kernel(const int32_t* __restrict__ nbr, const int32_t* __restrict__ cnt,
                                 int n, int K, int* __restrict__ deg) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)n * K) return;
  const int i = int(e / K), s = int(e % K);
  if (s >= row_count(cnt, i, K)) return;
  const int j = nbr[e];
  if ((unsigned)j < (unsigned)n) atomicAdd(&deg[j], 1);
}

// exclusive scan of deg[0..n) into ptr[0..n] by one CTA: tiles of 1024
// consecutive entries (coalesced), a warp-shuffle scan per tile, the running
// total carried between tiles; the next tile's loads are issued before the
// current tile's scan
__global__ void __launch_bounds__(1024) scan_one_cta_kernel(const int* __restrict__ deg, int n,
                                                           int* __restrict__ ptr) {
  __shared__ int wsum[32];
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  int carry = 0;
  int v = t < n ? deg[t] : 0;
  for (int base = 0; base < n; base += 1024) {
    const int nxt = base + 1024 + t;
    const int vn = nxt < n ? deg[nxt] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;
    }
    __syncthreads();
    if (base + t < n) ptr[base + t] = carry + (wid ? wsum[wid - 1] : 0) + x - v;
    carry += wsum[31];
    __syncthreads();   // wsum is rewritten by the next tile
    v = vn;
  }
  if (t == 0) ptr[n] = carry;
}

__global__ void in_fill_kernel(const int32_t* __restrict__ nbr, const int32_t* __restrict__ cnt,
                               int n, int K, const int* __restrict__ ptr, int* __restrict__ cursor,
                               int* __restrict__ in) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)n * K) return;
  const int i = int(e / K), s = int(e % K);
  if (s >= row_count(cnt, i, K)) return;
  const int j = nbr[e];
  if ((unsigned)j >= (unsigned)n) return;
  in[ptr[j] + atomicAdd(&cursor[j], 1)] = i;
}

// Sort every in-list ascending: a block-wide bitonic sort in shared memory
// up to kSortCap entries; a longer list (only for very dense systems) is
// ranked element by element through `scratch` (its entries are distinct).
__global__ void __launch_bounds__(256) in_sort_kernel(const int* __restrict__ ptr,
                                                      int* __restrict__ in,
                                                      int* __restrict__ scratch) {
  __shared__ int key[kSortCap];
  const int j = blockIdx.x;
  const int beg = ptr[j], len = ptr[j + 1] - beg;
  if (len <= 1) return;
  if (len <= kSortCap) {
    int m = 1;
    while (m < len) m <<= 1;
    for (int t = threadIdx.x; t < m; t += blockDim.x) key[t] = t < len ? in[beg + t] : INT_MAX;
    __syncthreads();
    for (int size = 2; size <= m; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int t = threadIdx.x; t < m; t += blockDim.x) {
          const int u = t ^ stride;
          if (u > t) {
            const bool up = (t & size) == 0;
            const int a = key[t], b = key[u];
            if ((a > b) == up) {
              key[t] = b;
              key[u] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int t = threadIdx.x; t < len; t += blockDim.x) in[beg + t] = key[t];
  } else {
    for (int t = threadIdx.x; t < len; t += blockDim.x) {
      const int v = in[beg + t];
      int rank = 0;
      for (int u = 0; u < len; ++u) rank += in[beg + u] < v;
      scratch[beg + rank] = v;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < len; t += blockDim.x) in[beg + t] = scratch[beg + t];
  }
}

// ---------------------------------------------------------------- steps 3, 4
struct BwdParams {
  const void* q;
  const void* k;
  const void* hp;
  const void* dm;
  const int32_t* nbr;    // [n][K]
  const int32_t* cnt;    // [n] or null
  const int* in_ptr;     // [n+1]
  const int* in;         // in-lists
  float* lse;            // [n][H]  log2-domain log-sum-exp of the logits
  float* delta;          // [n][H]
  float* dq;             // [n][H][dk]
  float* dk;             // [n][H][dk]
  float* dh;             // [n][D][C]
  const float* pos;
  const float* w1;
  const float* w2;
  const float* g;        // upstream gradient [n][D][C]
  const void* h;         // input features [n][D][C] (storage type)
  float* dpos;           // dL/dr [n][3], or null
  int n, H, dk_, K, cph;
  float qscale;          // log2(e) / sqrt(dk)
  float kscale;          // 1 / sqrt(dk)
  EaasTable tab;
  GenTable gen;
};

// dL/dr of one atom from the coupling values <g_c, T(x_c; r)> of all its
// channels c, with g and x staged in shared memory ([D][C] each) and the
// warp's Wigner-D scratch Dsm.  Every lane takes channels lane, lane + 32, ...;
// the warp reduces; the result is valid in every lane.
template <int L, int C, typename WFn>
__device__ __forceinline__ void atom_position_grad(const float* gs, const float* xs, float* Dsm,
                                                   const float (&r)[3], const EaasTable& tab,
                                                   const GenTable& gen, WFn wgt, int lane,
                                                   float (&out)[3]) {
  constexpr int D = (L + 1) * (L + 1);
  const float rho = sqrtf(r[0] * r[0] + r[1] * r[1] + r[2] * r[2]);
  out[0] = out[1] = out[2] = 0.f;
  if (rho > 0.f) {
    float Q[9];
    alignment_rotation(r[0], r[1], r[2], Q);
    wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
    __syncwarp();
    float rpow[L + 1], drpow[L + 1];
    rpow[0] = 1.f;
    drpow[0] = 0.f;
#pragma unroll
    for (int l = 1; l <= L; ++l) {
      rpow[l] = rpow[l - 1] * rho;
      drpow[l] = float(l) * rpow[l - 1];
    }
    float dr = 0.f, tx = 0.f, ty = 0.f;
    for (int c = lane; c < C; c += 32) {
      float g[D], x[D];
#pragma unroll
      for (int d = 0; d < D; ++d) {
        g[d] = gs[d * C + c];
        x[d] = xs[d * C + c];
      }
      coupling_grad_channel<L>(g, x, Dsm, rpow, drpow, tab, gen, [&](int pp) { return wgt(pp, c); },
                               dr, tx, ty);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dr += __shfl_xor_sync(0xffffffffu, dr, o);
      tx += __shfl_xor_sync(0xffffffffu, tx, o);
      ty += __shfl_xor_sync(0xffffffffu, ty, o);
    }
    // grad = Q ( -ty / rho, tx / rho, dr ): back from the aligned frame
    const float v0 = -ty / rho, v1 = tx / rho, v2 = dr;
#pragma unroll
    for (int a = 0; a < 3; ++a) out[a] = Q[3 * a] * v0 + Q[3 * a + 1] * v1 + Q[3 * a + 2] * v2;
  } else {
    // at r = 0 only degree-1 solid harmonics have a gradient, and R^1 is
    // linear: the derivative along axis a is the coupling at r = e_a with
    // the degree-1 paths alone, at unit weight
    float rpow1[L + 1];
#pragma unroll
    for (int l = 0; l <= L; ++l) rpow1[l] = l == 1 ? 1.f : 0.f;
    for (int a = 0; a < 3; ++a) {
      float Q[9];
      alignment_rotation(a == 0 ? 1.f : 0.f, a == 1 ? 1.f : 0.f, a == 2 ? 1.f : 0.f, Q);
      __syncwarp();
      wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
      __syncwarp();
      float s = 0.f;
      for (int c = lane; c < C; c += 32) {
        float g[D], t[D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
          g[d] = gs[d * C + c];
          t[d] = xs[d * C + c];
        }
        eaas_channel<L>(t, Dsm, rpow1, tab, [&](int pp) { return wgt(pp, c); },
                        [&](int d, float v) { s = fmaf(g[d], v, s); });
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      out[a] = s;
    }
  }
}

// sum over the lanes whose value chunks belong to the same head: the bits of
// the lane index inside a head's chunks (below cph) and the component bits
// (CPW and above)
template <int CPW>
__device__ __forceinline__ float head_sum(float v, int cph) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
    if (o < cph || o >= CPW) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int L, int C, typename T>
struct BwdLayout {
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int NCH = D * C / 8;          // 8-element chunks per row
  static constexpr int TPL = (NCH + 31) / 32;    // chunks per lane
  static constexpr int CPW = C / 8;              // chunks per component
  static_assert(32 % CPW == 0, "C/8 must divide 32");
  // Past 5 chunks per lane (lmax 3 with 128 channels) the warp's own row
  // (dm_i in the target pass, h'_j in the source pass) waits in the warp's
  // shared-memory slice instead of registers, and the kernel takes the whole
  // register file (one CTA per SM): three register rows of 64 floats would
  // spill.
  static constexpr bool OWN_SMEM = TPL > 5;
  static constexpr int MINB = OWN_SMEM ? 1 : 3;
};

// this lane's chunks of a row into a warp's shared-memory slice (float32)
template <int NCH, typename T>
__device__ __forceinline__ void stage_row(const T* __restrict__ row, float* own, int lane) {
  for (int q = lane; q < NCH; q += 32) {
    Chunk8<T> c;
    c.load(row + 8 * q);
    float v[8];
    c.to_f32(v);
#pragma unroll
    for (int e = 0; e < 8; ++e) own[8 * q + e] = v[e];
  }
}
// per-lane partial dot product of a staged row and a register row
template <int TPL, int NCH>
__device__ __forceinline__ float chunk_dot_smem(const float* own, const float (&b)[TPL][8],
                                                int lane) {
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    const int q = lane + 32 * t;
    if (q < NCH)
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(own[8 * q + e], b[t][e], s);
  }
  return s;
}

// per-lane partial dot product of two rows held as chunks
template <int TPL, int NCH>
__device__ __forceinline__ float chunk_dot(const float (&a)[TPL][8], const float (&b)[TPL][8],
                                           int lane) {
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < TPL; ++t)
    if (lane + 32 * t < NCH)
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(a[t][e], b[t][e], s);
  return s;
}

template <int TPL, int NCH, typename T>
__device__ __forceinline__ void load_row(const T* __restrict__ row, float (&v)[TPL][8], int lane) {
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    const int q = lane + 32 * t;
    Chunk8<T> c;
    if (q < NCH) c.load(row + 8 * q);
    else c.zero();
    c.to_f32(v[t]);
  }
}

// Step 3: one warp per target.
template <int L, int C, typename T>
__global__ void __launch_bounds__(kBwdWarps * 32, BwdLayout<L, C, T>::MINB)
attn_bwd_target_kernel(const __grid_constant__ BwdParams p) {
  using Ly = BwdLayout<L, C, T>;
  constexpr int D = Ly::D, NCH = Ly::NCH, TPL = Ly::TPL, CPW = Ly::CPW;
  constexpr bool OWN_SMEM = Ly::OWN_SMEM;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (i >= p.n) return;   // whole warp
  const T* __restrict__ qp = static_cast<const T*>(p.q);
  const T* __restrict__ kp = static_cast<const T*>(p.k);
  const float* __restrict__ hp = static_cast<const float*>(p.hp);
  const float* __restrict__ dmp = static_cast<const float*>(p.dm);
  const int hdk = p.H * p.dk_;
  const int kch = hdk >> 3;
  const int G = p.dk_ >> 3;
  const int head = ((lane % CPW) * 8 * p.H) / C;

  float qv[8];
  {
    Chunk8<T> qc;
    if (lane < kch) qc.load(qp + (size_t)i * hdk + 8 * lane);
    else qc.zero();
    qc.to_f32(qv);
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] *= p.qscale;
  }
  auto logit = [&](int j) {   // log2-domain logit of this lane's head
    float kf[8];
    Chunk8<T> kc;
    if (lane < kch) kc.load(kp + (size_t)j * hdk + 8 * lane);
    else kc.zero();
    kc.to_f32(kf);
    float sp = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sp = fmaf(qv[e], kf[e], sp);
    for (int o = 1; o < G; o <<= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    return __shfl_sync(0xffffffffu, sp, head * G);
  };
  const long long beg = (long long)i * p.K;
  const long long end = beg + row_count(p.cnt, i, p.K);

  // sweep 1 (key rows only): the log-sum-exp of the logits, online
  float mx = -INFINITY, z = 0.f;
  for (long long s = beg; s < end; ++s) {
    const int j = p.nbr[s];
    if ((unsigned)j >= (unsigned)p.n) continue;
    const float sl = logit(j);
    if (sl > mx) {
      z = z * exp2f(mx - sl) + 1.f;
      mx = sl;
    } else {
      z += exp2f(sl - mx);
    }
  }
  const float lse = z > 0.f ? mx + log2f(z) : -INFINITY;
  // dm_i: registers, or (OWN_SMEM) the warp's slice, where the epilogue's G_i goes later
  float* own = smem + (threadIdx.x >> 5) * (2 * D * C + wig_size(L));
  float dmv[OWN_SMEM ? 1 : TPL][8];
  if constexpr (OWN_SMEM) {
    stage_row<NCH>(dmp + (size_t)i * D * C, own, lane);
    __syncwarp();
  } else {
    load_row<TPL, NCH>(dmp + (size_t)i * D * C, dmv, lane);
  }

  // sweep 2 (key and value rows): with the exact weights alpha_ij,
  //   m_i = sum alpha h'_j, Delta_i = sum alpha dalpha,
  //   A = sum alpha dalpha k_j, B = sum alpha k_j, and dq_i = (A - Delta B) / sqrt(dk)
  // (Delta is constant over the sum, so sum alpha (dalpha - Delta) k = A - Delta B)
  float acc[TPL][8];
#pragma unroll
  for (int t = 0; t < TPL; ++t)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[t][e] = 0.f;
  float delta = 0.f;
  float qa[8], qb[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qa[e] = qb[e] = 0.f;
  const int khead = lane < kch ? lane / G : 0;   // head of this lane's key chunk
  for (long long s = beg; s < end; ++s) {
    const int j = p.nbr[s];
    if ((unsigned)j >= (unsigned)p.n) continue;
    const float a = exp2f(logit(j) - lse);
    float hv[TPL][8];
    load_row<TPL, NCH>(hp + (size_t)j * D * C, hv, lane);
    float dot;
    if constexpr (OWN_SMEM) dot = chunk_dot_smem<TPL, NCH>(own, hv, lane);
    else dot = chunk_dot<TPL, NCH>(dmv, hv, lane);
    const float da = head_sum<CPW>(dot, p.cph);
    delta = fmaf(a, da, delta);
#pragma unroll
    for (int t = 0; t < TPL; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[t][e] = fmaf(a, hv[t][e], acc[t][e]);
    const float ak = __shfl_sync(0xffffffffu, a, khead * p.cph);
    const float adk = __shfl_sync(0xffffffffu, a * da, khead * p.cph);
    if (lane < kch) {
      float kf[8];
      Chunk8<T> kc;
      kc.load(kp + (size_t)j * hdk + 8 * lane);
      kc.to_f32(kf);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        qa[e] = fmaf(adk, kf[e], qa[e]);
        qb[e] = fmaf(ak, kf[e], qb[e]);
      }
    }
  }
  if (lane < CPW && lane % p.cph == 0) {
    p.lse[(size_t)i * p.H + head] = lse;
    p.delta[(size_t)i * p.H + head] = delta;
  }
  const float dkh = __shfl_sync(0xffffffffu, delta, khead * p.cph);
  float dqv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) dqv[e] = fmaf(-dkh, qb[e], qa[e]);
  if (lane < kch) {
    float* o = p.dq + (size_t)i * hdk + 8 * lane;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = dqv[e] * p.kscale;
  }
  if (p.dpos) {
    // the target coupling's part of dL/dr_i: g = G_i, x = m_i
    constexpr int WS = wig_size(L);
    float* gs = own;              // (OWN_SMEM: dm_i is no longer read)
    float* xs = gs + D * C;
    float* Dsm = xs + D * C;
    __syncwarp();
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      const int q = lane + 32 * t;
      if (q < NCH)
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[8 * q + e] = acc[t][e];
    }
    for (int e = lane; e < D * C; e += 32) gs[e] = p.g[(size_t)i * D * C + e];
    __syncwarp();
    const float r[3] = {p.pos[3 * i], p.pos[3 * i + 1], p.pos[3 * i + 2]};
    float gr[3];
    atom_position_grad<L, C>(gs, xs, Dsm, r, p.tab, p.gen,
                             [&](int pp, int c) { return __ldg(p.w2 + pp * C + c); }, lane, gr);
    if (lane == 0) {
      p.dpos[3 * i] = gr[0];
      p.dpos[3 * i + 1] = gr[1];
      p.dpos[3 * i + 2] = gr[2];
    }
  }
}

// Step 4: one warp per source atom over its in-list, then the adjoint of the
// source coupling in the epilogue.
template <int L, int C, typename T>
__global__ void __launch_bounds__(kBwdWarps * 32, BwdLayout<L, C, T>::MINB)
attn_bwd_source_kernel(const __grid_constant__ BwdParams p) {
  using Ly = BwdLayout<L, C, T>;
  constexpr int D = Ly::D, NCH = Ly::NCH, TPL = Ly::TPL, CPW = Ly::CPW;
  constexpr bool OWN_SMEM = Ly::OWN_SMEM;
  constexpr int WS = wig_size(L);
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int j = blockIdx.x * kBwdWarps + wib;
  if (j >= p.n) return;   // whole warp
  const T* __restrict__ qp = static_cast<const T*>(p.q);
  const T* __restrict__ kp = static_cast<const T*>(p.k);
  const float* __restrict__ hp = static_cast<const float*>(p.hp);
  const float* __restrict__ dmp = static_cast<const float*>(p.dm);
  const int hdk = p.H * p.dk_;
  const int kch = hdk >> 3;
  const int G = p.dk_ >> 3;
  const int head = ((lane % CPW) * 8 * p.H) / C;
  const int khead = lane < kch ? lane / G : 0;

  float kv[8];
  {
    Chunk8<T> kc;
    if (lane < kch) kc.load(kp + (size_t)j * hdk + 8 * lane);
    else kc.zero();
    kc.to_f32(kv);
  }
  // h'_j: registers, or (OWN_SMEM) the warp's slice, where the epilogue's dh'_j goes later
  float* gbuf = smem + wib * (D * C + WS + (p.dpos ? D * C : 0));
  float hv[OWN_SMEM ? 1 : TPL][8];
  if constexpr (OWN_SMEM) {
    stage_row<NCH>(hp + (size_t)j * D * C, gbuf, lane);
    __syncwarp();
  } else {
    load_row<TPL, NCH>(hp + (size_t)j * D * C, hv, lane);
  }
  float dhp[TPL][8];
#pragma unroll
  for (int t = 0; t < TPL; ++t)
#pragma unroll
    for (int e = 0; e < 8; ++e) dhp[t][e] = 0.f;
  float dkv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) dkv[e] = 0.f;

  const int b = p.in_ptr[j], e_ = p.in_ptr[j + 1];
  for (int s = b; s < e_; ++s) {
    const int i = p.in[s];
    if ((unsigned)i >= (unsigned)p.n) continue;
    float qf[8];
    {
      Chunk8<T> qc;
      if (lane < kch) qc.load(qp + (size_t)i * hdk + 8 * lane);
      else qc.zero();
      qc.to_f32(qf);
    }
    float sp = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sp = fmaf(qf[e] * p.qscale, kv[e], sp);
    for (int o = 1; o < G; o <<= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    const float sl = __shfl_sync(0xffffffffu, sp, head * G);
    const float a = exp2f(sl - __ldg(p.lse + (size_t)i * p.H + head));
    float dmv[TPL][8];
    load_row<TPL, NCH>(dmp + (size_t)i * D * C, dmv, lane);
    float dot;
    if constexpr (OWN_SMEM) dot = chunk_dot_smem<TPL, NCH>(gbuf, dmv, lane);
    else dot = chunk_dot<TPL, NCH>(dmv, hv, lane);
    const float da = head_sum<CPW>(dot, p.cph);
    const float ds = a * (da - __ldg(p.delta + (size_t)i * p.H + head));
#pragma unroll
    for (int t = 0; t < TPL; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) dhp[t][e] = fmaf(a, dmv[t][e], dhp[t][e]);
    const float dsk = __shfl_sync(0xffffffffu, ds, khead * p.cph);
#pragma unroll
    for (int e = 0; e < 8; ++e) dkv[e] = fmaf(dsk, qf[e], dkv[e]);
  }
  if (lane < kch) {
    float* o = p.dk + (size_t)j * hdk + 8 * lane;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = dkv[e] * p.kscale;
  }

  // epilogue: dh_j = T*(dh'_j; r_j, w1), one channel per lane at a time
  float* Dsm = gbuf + D * C;
  __syncwarp();                   // (OWN_SMEM: h'_j is no longer read)
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    const int q = lane + 32 * t;
    if (q < NCH)
#pragma unroll
      for (int e = 0; e < 8; ++e) gbuf[8 * q + e] = dhp[t][e];
  }
  float Q[9];
  const float r = alignment_rotation(p.pos[3 * j], p.pos[3 * j + 1], p.pos[3 * j + 2], Q);
  float rpow[L + 1];
  rpow[0] = 1.f;
#pragma unroll
  for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
  wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
  __syncwarp();
  float* o = p.dh + (size_t)j * D * C;
  for (int c = lane; c < C; c += 32) {
    float x[D];
#pragma unroll
    for (int d = 0; d < D; ++d) x[d] = gbuf[d * C + c];
    eaas_channel_adjoint<L>(x, Dsm, rpow, p.tab, [&](int pp) { return __ldg(p.w1 + pp * C + c); },
                            [&](int d, float v) { o[d * C + c] = v; });
  }
  if (p.dpos) {
    // the source coupling's part of dL/dr_j: g = dh'_j, x = h_j, added to the
    // target part the target pass wrote
    float* xs = Dsm + WS;
    const T* hr = static_cast<const T*>(p.h) + (size_t)j * D * C;
    for (int e = lane; e < D * C; e += 32) xs[e] = load_one<T>(hr + e);
    __syncwarp();
    const float r[3] = {p.pos[3 * j], p.pos[3 * j + 1], p.pos[3 * j + 2]};
    float gr[3];
    atom_position_grad<L, C>(gbuf, xs, Dsm, r, p.tab, p.gen,
                             [&](int pp, int c) { return __ldg(p.w1 + pp * C + c); }, lane, gr);
    if (lane == 0) {
      p.dpos[3 * j] += gr[0];
      p.dpos[3 * j + 1] += gr[1];
      p.dpos[3 * j + 2] += gr[2];
    }
  }
}

// dL/dr of every atom when the attention gradients come from the tiled
// passes: one warp per atom adds the target coupling's part (g = G_a,
// x = m_a, weights w2) and the source coupling's part (g = dh'_a, x = h_a,
// weights w1).
struct PosGradParams {
  const float* g;     // upstream gradient [n][D][C]
  const float* m;     // m [n][D][C]
  const float* dhp;   // dL/dh' [n][D][C]
  const void* h;      // input features [n][D][C] (storage type)
  const float* pos;
  const float* w1;
  const float* w2;
  float* dpos;
  int n;
  EaasTable tab;
  GenTable gen;
};

constexpr int kPgWarps = 8;

// One warp per atom; both parts share the atom's rotation and Wigner-D, and
// every lane reads its channels' columns straight from global memory (lanes
// take consecutive channels: coalesced).
template <int L, int C, typename T>
__global__ void __launch_bounds__(kPgWarps * 32) position_grad_kernel(const __grid_constant__ PosGradParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int WS = wig_size(L);
  __shared__ float Dall[kPgWarps][WS];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int a = blockIdx.x * kPgWarps + wib;
  if (a >= p.n) return;   // whole warp
  float* Dsm = Dall[wib];
  const float* Gr = p.g + (size_t)a * D * C;
  const float* Mr = p.m + (size_t)a * D * C;
  const float* Sr = p.dhp + (size_t)a * D * C;
  const T* Xr = static_cast<const T*>(p.h) + (size_t)a * D * C;
  const float r0 = p.pos[3 * a], r1 = p.pos[3 * a + 1], r2 = p.pos[3 * a + 2];
  const float rho = sqrtf(r0 * r0 + r1 * r1 + r2 * r2);
  float out[3];
  if (rho > 0.f) {
    float Q[9];
    alignment_rotation(r0, r1, r2, Q);
    wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
    __syncwarp();
    float rpow[L + 1], drpow[L + 1];
    rpow[0] = 1.f;
    drpow[0] = 0.f;
#pragma unroll
    for (int l = 1; l <= L; ++l) {
      rpow[l] = rpow[l - 1] * rho;
      drpow[l] = float(l) * rpow[l - 1];
    }
    float dr = 0.f, tx = 0.f, ty = 0.f;
    for (int c = lane; c < C; c += 32) {
      float g[D], x[D];
      // the target coupling's part: g = G_a, x = m_a, weights w2
#pragma unroll
      for (int d = 0; d < D; ++d) {
        g[d] = __ldg(Gr + d * C + c);
        x[d] = __ldg(Mr + d * C + c);
      }
      coupling_grad_channel<L>(g, x, Dsm, rpow, drpow, p.tab, p.gen,
                               [&](int pp) { return __ldg(p.w2 + pp * C + c); }, dr, tx, ty);
      // the source coupling's part: g = dh'_a, x = h_a, weights w1
#pragma unroll
      for (int d = 0; d < D; ++d) {
        g[d] = __ldg(Sr + d * C + c);
        x[d] = load_one<T>(Xr + d * C + c);
      }
      coupling_grad_channel<L>(g, x, Dsm, rpow, drpow, p.tab, p.gen,
                               [&](int pp) { return __ldg(p.w1 + pp * C + c); }, dr, tx, ty);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dr += __shfl_xor_sync(0xffffffffu, dr, o);
      tx += __shfl_xor_sync(0xffffffffu, tx, o);
      ty += __shfl_xor_sync(0xffffffffu, ty, o);
    }
    // grad = Q ( -ty / rho, tx / rho, dr ): back from the aligned frame
    const float v0 = -ty / rho, v1 = tx / rho, v2 = dr;
#pragma unroll
    for (int e = 0; e < 3; ++e) out[e] = Q[3 * e] * v0 + Q[3 * e + 1] * v1 + Q[3 * e + 2] * v2;
  } else {
    // at r = 0: the derivative along axis e is the coupling at r = e_e with
    // the degree-1 paths alone (R^1 is linear), both parts
    float rpow1[L + 1];
#pragma unroll
    for (int l = 0; l <= L; ++l) rpow1[l] = l == 1 ? 1.f : 0.f;
    for (int e = 0; e < 3; ++e) {
      float Q[9];
      alignment_rotation(e == 0 ? 1.f : 0.f, e == 1 ? 1.f : 0.f, e == 2 ? 1.f : 0.f, Q);
      __syncwarp();
      wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
      __syncwarp();
      float sum = 0.f;
      for (int c = lane; c < C; c += 32) {
        float t[D];
#pragma unroll
        for (int d = 0; d < D; ++d) t[d] = __ldg(Mr + d * C + c);
        eaas_channel<L>(t, Dsm, rpow1, p.tab, [&](int pp) { return __ldg(p.w2 + pp * C + c); },
                        [&](int d, float v) { sum = fmaf(__ldg(Gr + d * C + c), v, sum); });
#pragma unroll
        for (int d = 0; d < D; ++d) t[d] = load_one<T>(Xr + d * C + c);
        eaas_channel<L>(t, Dsm, rpow1, p.tab, [&](int pp) { return __ldg(p.w1 + pp * C + c); },
                        [&](int d, float v) { sum = fmaf(__ldg(Sr + d * C + c), v, sum); });
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      out[e] = sum;
    }
  }
  if (lane == 0) {
    p.dpos[3 * a] = out[0];
    p.dpos[3 * a + 1] = out[1];
    p.dpos[3 * a + 2] = out[2];
  }
}

template <int L, typename T>
int launch_position_grad(const PosGradParams& p, cudaStream_t st) {
  position_grad_kernel<L, 128, T><<<(p.n + kPgWarps - 1) / kPgWarps, kPgWarps * 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

template <int L, int C, typename T>
int launch_attn_bwd(const BwdParams& p, cudaStream_t st) {
  constexpr int D = (L + 1) * (L + 1);
  const int grid = (p.n + kBwdWarps - 1) / kBwdWarps;
  // per warp: G_i, m_i and a Wigner-D scratch when dL/dr is wanted (the first
  // D * C floats also hold dm_i when the layout keeps it in shared memory)
  const size_t tshm = (p.dpos || BwdLayout<L, C, T>::OWN_SMEM)
                          ? size_t(kBwdWarps) * (2 * D * C + wig_size(L)) * sizeof(float) : 0;
  auto tkern = attn_bwd_target_kernel<L, C, T>;
  if (tshm > 48 * 1024 &&
      cudaFuncSetAttribute(tkern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tshm)) != cudaSuccess)
    return EGAT_ERR_CUDA;
  tkern<<<grid, kBwdWarps * 32, tshm, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return EGAT_ERR_CUDA;
  // per warp: dh'_j, the Wigner-D scratch and (dL/dr) h_j
  const size_t shmem =
      size_t(kBwdWarps) * (D * C + wig_size(L) + (p.dpos ? D * C : 0)) * sizeof(float);
  auto kern = attn_bwd_source_kernel<L, C, T>;
  if (shmem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shmem)) != cudaSuccess)
    return EGAT_ERR_CUDA;
  kern<<<grid, kBwdWarps * 32, shmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

template <int L, typename T>
int dispatch_c(const BwdParams& p, int C, cudaStream_t st) {
  switch (C) {
    case 16: return launch_attn_bwd<L, 16, T>(p, st);
    case 32: return launch_attn_bwd<L, 32, T>(p, st);
    case 64: return launch_attn_bwd<L, 64, T>(p, st);
    case 128: return launch_attn_bwd<L, 128, T>(p, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

template <int L, typename T, bool TF32 = false>
int launch_adjoint(const egat_shape& s, const float* g, const float* pos, const float* w, void* out,
                   cudaStream_t st) {
  const int grid = (s.n + kBwdWarps - 1) / kBwdWarps;
  adjoint_coupling_kernel<L, T, TF32><<<grid, kBwdWarps * 32, 0, st>>>(g, pos, w, static_cast<T*>(out),
                                                                      s.n, s.C, eaas_table(L));
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

template <int L, typename T, bool TF32 = false>
int launch_adjoint_planned(const egat_shape& s, const float* g, const void* plan, const float* w, void* out,
                           cudaStream_t st) {
  const PlanView pv = plan_view(const_cast<void*>(plan), s.n, s.K, s.lmax);
  const long long items = (long long)pv.tiles * kTileM;
  const long long grid = (items + kBwdWarps - 1) / kBwdWarps;
  adjoint_planned_kernel<L, T, TF32><<<unsigned(grid), kBwdWarps * 32, 0, st>>>(
      g, pv.rec, items, w, static_cast<T*>(out), s.n, s.C, eaas_table(L));
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// host, double precision: the Ivanic–Ruedenberg recursion of wigner_build,
// for the rotation generators below
double ir_entry_host(int l, int m, int mp, const double* D1, const double* Dp) {
  const int wp = 2 * l - 1;
  auto r1 = [&](int i, int j) { return D1[(i + 1) * 3 + (j + 1)]; };
  auto rp = [&](int a, int b) { return Dp[(a + l - 1) * wp + (b + l - 1)]; };
  auto P = [&](int i, int a, int b) -> double {
    if (b == l) return r1(i, 1) * rp(a, l - 1) - r1(i, -1) * rp(a, -l + 1);
    if (b == -l) return r1(i, 1) * rp(a, -l + 1) + r1(i, -1) * rp(a, l - 1);
    return r1(i, 0) * rp(a, b);
  };
  const double d = (std::abs(mp) == l) ? double((2 * l) * (2 * l - 1)) : double((l + mp) * (l - mp));
  const int am = std::abs(m);
  double val = 0.0;
  if (am < l) val += std::sqrt(double((l + m) * (l - m)) / d) * P(0, m, mp);
  {
    const double v = 0.5 * std::sqrt(double((m == 0 ? 2 : 1) * (l + am - 1) * (l + am)) / d) *
                     (m == 0 ? -1.0 : 1.0);
    double V;
    if (m == 0) V = P(1, 1, mp) + P(-1, -1, mp);
    else if (m > 0) V = P(1, m - 1, mp) * (m == 1 ? std::sqrt(2.0) : 1.0) - (m == 1 ? 0.0 : P(-1, -m + 1, mp));
    else V = (m == -1 ? 0.0 : P(1, m + 1, mp)) + P(-1, -m - 1, mp) * (m == -1 ? std::sqrt(2.0) : 1.0);
    val += v * V;
  }
  if (m != 0 && am < l - 1) {
    const double w = -0.5 * std::sqrt(double((l - am - 1) * (l - am)) / d);
    const double W = (m > 0) ? (P(1, m + 1, mp) + P(-1, -m - 1, mp)) : (P(1, m - 1, mp) - P(-1, -m + 1, mp));
    val += w * W;
  }
  return val;
}

void wigner_host(const double (&Q)[9], double* D) {
  D[0] = 1.0;
  for (int e = 0; e < 9; ++e) D[wig_off(1) + e] = Q[wig1_src(e)];
  for (int l = 2; l <= kMaxL; ++l) {
    const int w = 2 * l + 1;
    for (int e = 0; e < w * w; ++e)
      D[wig_off(l) + e] = ir_entry_host(l, e / w - l, e % w - l, D + wig_off(1), D + wig_off(l - 1));
  }
}

// J_a = dD(R_a(t))/dt at t = 0, by central differences of the recursion in
// double precision (step 1e-5: error ~1e-10, far below float rounding)
GenTable make_gen_table() {
  GenTable g;
  const double h = 1e-5;
  for (int a = 0; a < 3; ++a) {
    double Dp[wig_size(kMaxL)], Dm[wig_size(kMaxL)];
    for (int sgn = 0; sgn < 2; ++sgn) {
      const double t = sgn == 0 ? h : -h;
      const double c = std::cos(t), s_ = std::sin(t);
      double Q[9] = {1, 0, 0, 0, 1, 0, 0, 0, 1};
      const int i = (a + 1) % 3, j = (a + 2) % 3;   // the plane the rotation turns
      Q[i * 3 + i] = c;
      Q[i * 3 + j] = -s_;
      Q[j * 3 + i] = s_;
      Q[j * 3 + j] = c;
      wigner_host(Q, sgn == 0 ? Dp : Dm);
    }
    for (int e = 0; e < wig_size(kMaxL); ++e) g.J[a][e] = float((Dp[e] - Dm[e]) / (2 * h));
  }
  return g;
}

const GenTable& gen_table() {
  static std::once_flag once;
  static GenTable g;
  std::call_once(once, [] { g = make_gen_table(); });
  return g;
}

struct BwdWs {
  BwdTcWs tc;   // the tiled path's part (tiled shapes only)
  void* hp;
  void* dm;
  int* deg;
  int* ptr;
  int* cursor;
  int* in;
  int* scratch;
  float* lse;
  float* delta;
  size_t bytes;
};

BwdWs bwd_ws(const egat_shape& s, void* base) {
  const size_t D = size_t(s.lmax + 1) * (s.lmax + 1);
  const size_t row = D * s.C * sizeof(float);   // h' and dm in float32
  const size_t n = size_t(s.n), E = size_t(s.n) * s.K;
  BwdWs w;
  char* b = static_cast<char*>(base);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    void* ptr = b ? b + o : nullptr;
    o += a256(bytes);
    return ptr;
  };
  w.hp = take(n * row);
  w.dm = take(n * row);
  w.deg = static_cast<int*>(take(n * 4));
  w.ptr = static_cast<int*>(take((n + 1) * 4));
  w.cursor = static_cast<int*>(take(n * 4));
  w.in = static_cast<int*>(take(E * 4));
  w.scratch = static_cast<int*>(take(E * 4));
  w.lse = static_cast<float*>(take(n * s.H * 4));
  w.delta = static_cast<float*>(take(n * s.H * 4));
  if (bwd_tc_supported(s)) {
    void* t = take(bwd_tc_ws_bytes(s));
    if (b) w.tc = bwd_tc_ws(s, t);
  }
  w.bytes = o;
  return w;
}

}  // namespace

size_t backward_ws_bytes(const egat_shape& s) { return bwd_ws(s, nullptr).bytes; }

int launch_exclusive_scan(const int* d_in, int n, int* d_out, cudaStream_t st) {
  scan_one_cta_kernel<<<1, 1024, 0, st>>>(d_in, n, d_out);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

// The tiled path (bwd_tc_supported): the forward plan (target tiles) first,
// whose tile records give every coupling below its rotations; h' in float32
// rounded to tf32 as it is stored, dm in float32 (rounded to tf32 where it
// enters a single tf32 product, split into tf32 hi + lo where it forms
// dL/dh'); the in-lists, then the statistics, target and source passes, the
// source coupling's adjoint and dL/dr.
template <int L>
int launch_backward_tiled(const egat_shape& s, const BwdWs& w, const void* d_h, const float* d_pos,
                          const void* d_q, const void* d_k, const int32_t* d_nbr,
                          const int32_t* d_cnt, const int32_t* d_order, const float* d_w1,
                          const float* d_w2, const float* d_g, float* d_dh, float* d_dq,
                          float* d_dk, float* d_dpos, cudaStream_t st) {
  float* hp = static_cast<float*>(w.hp);
  float* dm = static_cast<float*>(w.dm);
  // the forward plan first: its tile records give the source coupling its
  // rotations (the tile-staged kernel), then dL/dm
  int e = launch_build_plan(s.n, s.K, s.lmax, d_nbr, d_cnt, d_order, d_pos, w.tc.plan, st);
  if (e == EGAT_OK) e = launch_eaas_planned_tf32out(s, d_h, w.tc.plan, d_w1, hp, st);
  if (e == EGAT_OK) e = launch_adjoint_planned<L, float>(s, d_g, w.tc.plan, d_w2, dm, st);
  if (e != EGAT_OK) return e;
  // in-lists (unsorted: the source plan's union is ordered by its bitmap)
  if (cudaMemsetAsync(w.deg, 0, size_t(s.n) * 4, st) != cudaSuccess ||
      cudaMemsetAsync(w.cursor, 0, size_t(s.n) * 4, st) != cudaSuccess)
    return EGAT_ERR_CUDA;
  const long long E = (long long)s.n * s.K;
  const int eb = int((E + 255) / 256);
  in_degree_kernel<<<eb, 256, 0, st>>>(d_nbr, d_cnt, s.n, s.K, w.deg);
  scan_one_cta_kernel<<<1, 1024, 0, st>>>(w.deg, s.n, w.ptr);
  in_fill_kernel<<<eb, 256, 0, st>>>(d_nbr, d_cnt, s.n, s.K, w.ptr, w.cursor, w.in);
  if (cudaGetLastError() != cudaSuccess) return EGAT_ERR_CUDA;
  e = launch_backward_tc(s, w.tc, d_q, d_k, hp, dm, d_order, w.ptr, w.in, d_dq, d_dk, d_dpos != nullptr,
                         st);
  if (e == EGAT_OK) e = launch_adjoint_planned<L, float>(s, w.tc.dhp, w.tc.plan, d_w1, d_dh, st);
  if (e != EGAT_OK || !d_dpos) return e;
  PosGradParams pg;
  pg.g = d_g;
  pg.m = w.tc.m;
  pg.dhp = w.tc.dhp;
  pg.h = d_h;
  pg.pos = d_pos;
  pg.w1 = d_w1;
  pg.w2 = d_w2;
  pg.dpos = d_dpos;
  pg.n = s.n;
  pg.tab = eaas_table(s.lmax);
  pg.gen = gen_table();
  return launch_position_grad<L, __nv_bfloat16>(pg, st);
}

int launch_backward(const egat_shape& s, const void* d_h, const float* d_pos, const void* d_q,
                    const void* d_k, const int32_t* d_nbr, const int32_t* d_cnt,
                    const int32_t* d_order, const float* d_w1, const float* d_w2, const float* d_g,
                    void* d_ws, float* d_dh, float* d_dq, float* d_dk, float* d_dpos,
                    cudaStream_t st) {
  const BwdWs w = bwd_ws(s, d_ws);
  const bool bf = s.dtype == EGAT_BF16;
  if (bwd_tc_supported(s)) {
    switch (s.lmax) {
      case 1: return launch_backward_tiled<1>(s, w, d_h, d_pos, d_q, d_k, d_nbr, d_cnt, d_order, d_w1, d_w2, d_g, d_dh, d_dq, d_dk, d_dpos, st);
      case 2: return launch_backward_tiled<2>(s, w, d_h, d_pos, d_q, d_k, d_nbr, d_cnt, d_order, d_w1, d_w2, d_g, d_dh, d_dq, d_dk, d_dpos, st);
      case 3: return launch_backward_tiled<3>(s, w, d_h, d_pos, d_q, d_k, d_nbr, d_cnt, d_order, d_w1, d_w2, d_g, d_dh, d_dq, d_dk, d_dpos, st);
      default: return EGAT_ERR_UNSUPPORTED;
    }
  }
  // h' = source coupling (forward step 2), in float32
  int e = launch_eaas_source_f32out(s, d_h, d_pos, d_w1, static_cast<float*>(w.hp), st);
  if (e != EGAT_OK) return e;
  // step 1: dm = T*(G; r, w2)
  switch (s.lmax) {
    case 1: e = launch_adjoint<1, float>(s, d_g, d_pos, d_w2, w.dm, st); break;
    case 2: e = launch_adjoint<2, float>(s, d_g, d_pos, d_w2, w.dm, st); break;
    case 3: e = launch_adjoint<3, float>(s, d_g, d_pos, d_w2, w.dm, st); break;
    default: return EGAT_ERR_UNSUPPORTED;
  }
  if (e != EGAT_OK) return e;
  // step 2: in-lists
  if (cudaMemsetAsync(w.deg, 0, size_t(s.n) * 4, st) != cudaSuccess ||
      cudaMemsetAsync(w.cursor, 0, size_t(s.n) * 4, st) != cudaSuccess)
    return EGAT_ERR_CUDA;
  const long long E = (long long)s.n * s.K;
  const int eb = int((E + 255) / 256);
  in_degree_kernel<<<eb, 256, 0, st>>>(d_nbr, d_cnt, s.n, s.K, w.deg);
  scan_one_cta_kernel<<<1, 1024, 0, st>>>(w.deg, s.n, w.ptr);
  in_fill_kernel<<<eb, 256, 0, st>>>(d_nbr, d_cnt, s.n, s.K, w.ptr, w.cursor, w.in);
  in_sort_kernel<<<s.n, 256, 0, st>>>(w.ptr, w.in, w.scratch);
  if (cudaGetLastError() != cudaSuccess) return EGAT_ERR_CUDA;
  // steps 3, 4
  BwdParams p;
  p.q = d_q;
  p.k = d_k;
  p.hp = w.hp;
  p.dm = w.dm;
  p.nbr = d_nbr;
  p.cnt = d_cnt;
  p.in_ptr = w.ptr;
  p.in = w.in;
  p.lse = w.lse;
  p.delta = w.delta;
  p.dq = d_dq;
  p.dk = d_dk;
  p.dh = d_dh;
  p.pos = d_pos;
  p.w1 = d_w1;
  p.w2 = d_w2;
  p.g = d_g;
  p.h = d_h;
  p.dpos = d_dpos;
  p.gen = gen_table();
  p.n = s.n;
  p.H = s.H;
  p.dk_ = s.dk;
  p.K = s.K;
  p.cph = s.C / (8 * s.H);
  p.qscale = float(1.4426950408889634 / std::sqrt(double(s.dk)));
  p.kscale = float(1.0 / std::sqrt(double(s.dk)));
  p.tab = eaas_table(s.lmax);
  switch (s.lmax) {
    case 1: return bf ? dispatch_c<1, __nv_bfloat16>(p, s.C, st) : dispatch_c<1, float>(p, s.C, st);
    case 2: return bf ? dispatch_c<2, __nv_bfloat16>(p, s.C, st) : dispatch_c<2, float>(p, s.C, st);
    case 3: return bf ? dispatch_c<3, __nv_bfloat16>(p, s.C, st) : dispatch_c<3, float>(p, s.C, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

}  // namespace egat
