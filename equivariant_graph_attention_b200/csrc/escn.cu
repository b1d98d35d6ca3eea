// Edge-centric eSCN convolution: the comparison workload.
//
// "EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-Equivariant Graph Attention Transformers",
// section "eSCN卷积与SO(2)线性层": per edge, rotate the source's features by D(Q_ij) into the frame
// whose z axis is r_ij = r_j - r_i, apply an SO(2) linear layer that acts
// within each order m (mixing degrees; components with |m| > M_max dropped),
// rotate back, and sum the messages over the neighbour list:
//   out_i = sum_j D(Q_ij) SO2_W(D(Q_ij)^T h_j).
// Per channel c the layer is
//   y~^lo_0  = sum_li W0[lo][li][c] x~^li_0,
//   y~^lo_+m = sum_li W1_m[lo][li][c] x~^li_+m - W2_m[lo][li][c] x~^li_-m,
//   y~^lo_-m = sum_li W2_m[lo][li][c] x~^li_+m + W1_m[lo][li][c] x~^li_-m.
// This is the edge-centric formulation that the node-centric factorisation
// of "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.1 replaces: every
// edge needs its own Wigner-D matrices and two rotations of the whole
// neighbour row, where EAAS rotates each atom once.
//
// B200 mapping: one warp per target, targets in the graph builder's cell
// order so that concurrently resident warps share neighbour rows in L2.  Per
// edge the warp builds D^0..D^L of Q_ij cooperatively in its own slice of
// shared memory (Ivanic–Ruedenberg recursion, __syncwarp only); each lane
// owns CPL consecutive channels, holds them of the neighbour row and of the
// running sum in registers and reads the rotation entries and its channels'
// SO(2) weights from shared memory.  With 128 channels at lmax >= 2 the warp
// walks the neighbour list twice, 64 channels a pass, so that two CTAs fit an
// SM without spilling (four channels a lane would need more than 128
// registers).  Messages are summed on chip; nothing per edge reaches memory.
#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kEscnWarps = 8;

struct EscnParams {
  const void* h;
  const float* pos;
  const int32_t* nbr;
  const int32_t* cnt;
  const int32_t* order;
  const float* w;     // [nw][C]
  float* out;         // [n][D][C]
  int n, K, C, nw, mmax;
};

constexpr int escn_num_weights(int L, int mmax) {
  int nw = (L + 1) * (L + 1);
  for (int m = 1; m <= mmax; ++m) nw += 2 * (L + 1 - m) * (L + 1 - m);
  return nw;
}
// first weight row of the W1_m block (W2_m follows it)
constexpr int escn_block(int L, int m) {
  int off = (L + 1) * (L + 1);
  for (int q = 1; q < m; ++q) off += 2 * (L + 1 - q) * (L + 1 - q);
  return off;
}

// M is the truncation order M_max (compile time, so the SO(2) layer is
// straight-line code); two CTAs per SM below lmax 3, one at lmax 3 (whose
// 16-component rows need more than 128 registers).
template <int L, int M, typename T, int CPL, int PASSES>
__global__ void __launch_bounds__(kEscnWarps * 32, L >= 3 ? 1 : 2)
escn_conv_kernel(const __grid_constant__ EscnParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int WS = wig_size(L);
  extern __shared__ float smem[];
  float* sw = smem;                                  // [nw][C]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* Dw = smem + p.nw * p.C + warp * WS;         // this warp's D^0..D^L
  for (int e = tid; e < p.nw * p.C; e += blockDim.x) sw[e] = __ldg(p.w + e);
  __syncthreads();

  const int C = p.C;
  const T* h = static_cast<const T*>(p.h);
  const long long stride = (long long)gridDim.x * kEscnWarps;
  for (long long slot = (long long)blockIdx.x * kEscnWarps + warp; slot < p.n; slot += stride) {
    const int i = p.order ? p.order[slot] : int(slot);
    if ((unsigned)i >= (unsigned)p.n) continue;     // warp-uniform
#pragma unroll 1
    for (int pass = 0; pass < PASSES; ++pass) {
    const int c0 = (pass * 32 + lane) * CPL;
    const bool live = c0 < C;
    float acc[D][CPL];
#pragma unroll
    for (int d = 0; d < D; ++d)
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[d][k] = 0.f;
    const float xi = p.pos[3 * i], yi = p.pos[3 * i + 1], zi = p.pos[3 * i + 2];
    int cnt = p.cnt ? p.cnt[i] : p.K;
    cnt = cnt < 0 ? 0 : (cnt > p.K ? p.K : cnt);
    const int32_t* row = p.nbr + (long long)i * p.K;
    for (int e = 0; e < cnt; ++e) {
      const int j = row[e];
      if ((unsigned)j >= (unsigned)p.n) continue;   // warp-uniform
      float Q[9];
      alignment_rotation(p.pos[3 * j] - xi, p.pos[3 * j + 1] - yi, p.pos[3 * j + 2] - zi, Q);
      __syncwarp();                                 // the previous edge's readers are done
      wigner_build<L>(Q, Dw, lane, 32, [] { __syncwarp(); });
      if (!live) continue;
      // the neighbour's row, this lane's channels
      float x[D][CPL];
      const T* hr = h + (long long)j * D * C + c0;
#pragma unroll
      for (int d = 0; d < D; ++d)
#pragma unroll
        for (int k = 0; k < CPL; ++k) x[d][k] = load_one<T>(hr + d * C + k);
      // into the edge frame: x~^l = D^l^T x^l
      static_for<1, L + 1>([&](auto lc) {
        constexpr int l = decltype(lc)::value;
        constexpr int w = 2 * l + 1;
        const float* Dl = Dw + wig_off(l);
        float t[w][CPL];
#pragma unroll
        for (int a = 0; a < w; ++a)
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            float s = 0.f;
#pragma unroll
            for (int b = 0; b < w; ++b) s = fmaf(Dl[b * w + a], x[l * l + b][k], s);
            t[a][k] = s;
          }
#pragma unroll
        for (int a = 0; a < w; ++a)
#pragma unroll
          for (int k = 0; k < CPL; ++k) x[l * l + a][k] = t[a][k];
      });
      // SO(2) linear layer in the edge frame
      float y[D][CPL];
#pragma unroll
      for (int d = 0; d < D; ++d)
#pragma unroll
        for (int k = 0; k < CPL; ++k) y[d][k] = 0.f;
#pragma unroll
      for (int lo = 0; lo <= L; ++lo)
#pragma unroll
        for (int li = 0; li <= L; ++li) {
          const float* w0 = sw + (lo * (L + 1) + li) * C + c0;
#pragma unroll
          for (int k = 0; k < CPL; ++k)
            y[lo * lo + lo][k] = fmaf(w0[k], x[li * li + li][k], y[lo * lo + lo][k]);
#pragma unroll
          for (int m = 1; m <= M; ++m) {
            if (m > lo || m > li) continue;         // compile-time after unrolling
            const int nb = L + 1 - m;
            const int r = (lo - m) * nb + (li - m);
            const float* w1 = sw + (escn_block(L, m) + r) * C + c0;
            const float* w2 = sw + (escn_block(L, m) + nb * nb + r) * C + c0;
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
              const float xp = x[li * li + li + m][k], xm = x[li * li + li - m][k];
              y[lo * lo + lo + m][k] = fmaf(w1[k], xp, fmaf(-w2[k], xm, y[lo * lo + lo + m][k]));
              y[lo * lo + lo - m][k] = fmaf(w2[k], xp, fmaf(w1[k], xm, y[lo * lo + lo - m][k]));
            }
          }
        }
      // back to the global frame and into the sum: acc^l += D^l y~^l
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[0][k] += y[0][k];
      static_for<1, L + 1>([&](auto lc) {
        constexpr int l = decltype(lc)::value;
        constexpr int w = 2 * l + 1;
        const float* Dl = Dw + wig_off(l);
#pragma unroll
        for (int a = 0; a < w; ++a)
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            float s = acc[l * l + a][k];
#pragma unroll
            for (int b = 0; b < w; ++b) s = fmaf(Dl[a * w + b], y[l * l + b][k], s);
            acc[l * l + a][k] = s;
          }
      });
    }
    if (live) {
      float* o = p.out + (long long)i * D * C + c0;
#pragma unroll
      for (int d = 0; d < D; ++d)
#pragma unroll
        for (int k = 0; k < CPL; ++k) o[d * C + k] = acc[d][k];
    }
    }   // channel passes
  }
}

template <int L, int M, typename T>
int launch_escn_m(const EscnParams& p, cudaStream_t st) {
  const size_t shmem = (size_t(p.nw) * p.C + size_t(kEscnWarps) * wig_size(L)) * sizeof(float);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (p.n + kEscnWarps - 1) / kEscnWarps;
  const int grid = int(std::max<long long>(1, std::min<long long>(want, (long long)sms * 8)));
  switch (p.C) {
    case 32: escn_conv_kernel<L, M, T, 1, 1><<<grid, kEscnWarps * 32, shmem, st>>>(p); break;
    case 64: escn_conv_kernel<L, M, T, 2, 1><<<grid, kEscnWarps * 32, shmem, st>>>(p); break;
    case 128:
      if constexpr (L >= 2) escn_conv_kernel<L, M, T, 2, 2><<<grid, kEscnWarps * 32, shmem, st>>>(p);
      else escn_conv_kernel<L, M, T, 4, 1><<<grid, kEscnWarps * 32, shmem, st>>>(p);
      break;
    default: escn_conv_kernel<L, M, T, 1, 1><<<grid, kEscnWarps * 32, shmem, st>>>(p); break;   // C = 16
  }
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

template <int L, typename T>
int launch_escn_t(const EscnParams& p, cudaStream_t st) {
  switch (p.mmax) {
    case 0: return launch_escn_m<L, 0, T>(p, st);
    case 1: return launch_escn_m<L, 1, T>(p, st);
    case 2: if constexpr (L >= 2) return launch_escn_m<L, 2, T>(p, st); else return EGAT_ERR_ARG;
    case 3: if constexpr (L >= 3) return launch_escn_m<L, 3, T>(p, st); else return EGAT_ERR_ARG;
    default: return EGAT_ERR_ARG;
  }
}

}  // namespace

int escn_num_weights_host(int lmax, int mmax) { return escn_num_weights(lmax, mmax); }

int launch_escn_conv(const egat_shape& s, int mmax, const void* d_h, const float* d_pos,
                     const int32_t* d_nbr, const int32_t* d_cnt, const int32_t* d_order,
                     const float* d_w, float* d_out, cudaStream_t st) {
  EscnParams p;
  p.h = d_h;
  p.pos = d_pos;
  p.nbr = d_nbr;
  p.cnt = d_cnt;
  p.order = d_order;
  p.w = d_w;
  p.out = d_out;
  p.n = s.n;
  p.K = s.K;
  p.C = s.C;
  p.nw = escn_num_weights(s.lmax, mmax);
  p.mmax = mmax;
  const bool bf = s.dtype == EGAT_BF16;
  switch (s.lmax) {
    case 1: return bf ? launch_escn_t<1, __nv_bfloat16>(p, st) : launch_escn_t<1, float>(p, st);
    case 2: return bf ? launch_escn_t<2, __nv_bfloat16>(p, st) : launch_escn_t<2, float>(p, st);
    case 3: return bf ? launch_escn_t<3, __nv_bfloat16>(p, st) : launch_escn_t<3, float>(p, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

}  // namespace egat
