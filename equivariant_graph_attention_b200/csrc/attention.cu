// Step 3 (on-the-fly attention) and steps 3+4 fused (attention with the EAAS
// target coupling in the epilogue).
//
// [EX] = "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构": §3.1 (node-centric
// factorisation: m_i = sum_j alpha_ij h'_j, then ^h_i = m_i (x) R(r_i)), §3.2
// (online softmax with a running max and normaliser, each key/value loaded
// once, on-chip accumulation, one target per program, padded neighbours
// skipped).  [TS] = "E2Former-V2: On-the-Fly Equivariant Attention with
// Linear Activation Memory" §2.2 (invariant scalar logits, Eq. 6; streaming
// reduction; no N x K x H x D tensor in HBM).
//
// B200 design: one warp per target atom.  A neighbour's value row h'_j is
// D*C elements; lane l owns the 8-element chunks l, l+32, l+64, ... of that
// row (16-byte loads for bf16), so one warp-wide load moves 512 contiguous
// bytes.  With C/8 a divisor of 32 every chunk a lane owns lies in the same
// channel block, hence the same head, so each lane keeps one running max and
// normaliser.  The key row is H*dk elements: lane r < H*dk/8 loads chunk r,
// multiplies it with its register-resident slice of q_i and the dk/8 lanes of
// a head reduce by shuffles; every lane then fetches its own head's logit
// with one shuffle.  Neighbour indices are read four slots ahead and rows one
// slot ahead into two register buffers used in ping-pong, so the gathers
// overlap the arithmetic.  Accumulation uses the packed f32x2 FMA (two
// channels per instruction); the online-softmax reference maximum is raised
// lazily (only when a logit exceeds it by 2^8), which keeps the rescale of
// the accumulators off the per-edge path.  Nothing per edge is written.  The fused variant writes m_i / z to shared
// memory, rebuilds the target's Wigner-D matrices in shared memory, and lets
// each lane apply EAAS to its channels before writing ^h_i.
#include <cfloat>

#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kAttnWarps = 4;

struct AttnParams {
  const void* q;
  const void* k;
  const void* hp;
  const int32_t* nbr;   // PADDED: [n][K]; CSR: rowptr [n+1]
  const int32_t* cnt;   // PADDED: [n] or null; CSR: col
  const int32_t* order;
  float* out;
  const float* pos;
  const float* w2;
  int n, H, dk, K, mode;
  long long n_edges;
  float qscale;         // log2(e) / sqrt(dk)
  EaasTable tab;
};

template <int L, int C, typename T>
struct Frag {
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int NCH = D * C / 8;
  static constexpr int TPL = (NCH + 31) / 32;
  Chunk8<T> kc;
  Chunk8<T> hc[TPL];

  __device__ __forceinline__ void load(const T* __restrict__ k, const T* __restrict__ hp, int j,
                                       int lane, int kch, int hdk) {
    if (lane < kch) kc.load(k + (size_t)j * hdk + 8 * lane);
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      const int q = lane + 32 * t;
      if (q < NCH) hc[t].load(hp + (size_t)j * D * C + 8 * q);
    }
  }
};

template <int L, int C, typename T, bool FUSED>
__global__ void __launch_bounds__(kAttnWarps * 32)
otf_attention_kernel(const __grid_constant__ AttnParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int NCH = D * C / 8;          // 8-element chunks per value row
  constexpr int TPL = (NCH + 31) / 32;    // chunks per lane
  constexpr int CPW = C / 8;              // chunks per component (divides 32)
  static_assert(32 % CPW == 0, "C/8 must divide 32");
  extern __shared__ float smem[];

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int gw = blockIdx.x * kAttnWarps + wib;
  if (gw >= p.n) return;
  const int i = p.order ? p.order[gw] : gw;
  if ((unsigned)i >= (unsigned)p.n) return;

  const T* __restrict__ qp = static_cast<const T*>(p.q);
  const T* __restrict__ kp = static_cast<const T*>(p.k);
  const T* __restrict__ hp = static_cast<const T*>(p.hp);
  const int hdk = p.H * p.dk;
  const int kch = hdk >> 3;        // key chunks per row (<= 32)
  const int G = p.dk >> 3;         // lanes per head in the key row
  const int head = ((lane % CPW) * 8 * p.H) / C;
  const int src_lane = head * G;

  float qv[8];
  {
    Chunk8<T> qc;
    if (lane < kch) qc.load(qp + (size_t)i * hdk + 8 * lane);
    else qc.zero();
    qc.to_f32(qv);
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] *= p.qscale;
  }

  long long beg, end;
  if (p.mode == EGAT_GRAPH_PADDED) {
    beg = (long long)i * p.K;
    int c = p.cnt ? p.cnt[i] : p.K;
    c = c < 0 ? 0 : (c > p.K ? p.K : c);
    end = beg + c;
  } else {
    long long a = p.nbr[i], b = p.nbr[i + 1];
    a = a < 0 ? 0 : (a > p.n_edges ? p.n_edges : a);
    b = b < a ? a : (b > p.n_edges ? p.n_edges : b);
    beg = a;
    end = b;
  }
  const int32_t* __restrict__ idx = (p.mode == EGAT_GRAPH_PADDED) ? p.nbr : p.cnt;

  // accumulators as packed float pairs: acc[t][e] holds elements 2e, 2e+1 of chunk t
  f32x2 acc[TPL][4];
#pragma unroll
  for (int t = 0; t < TPL; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0ull;
  // Online softmax in the log2 domain.  mref is a running reference maximum
  // that is raised only when a logit exceeds it by more than kLazy, so the
  // O(D*C/32) rescale of the accumulators is rare; every weight is
  // 2^(s - mref) <= 2^kLazy and z, acc share the same reference, so m = acc / z
  // is the softmax average exactly as with the true running maximum.
  constexpr float kLazy = 8.f;
  float mref = -INFINITY, z = 0.f;

  auto valid = [&](int j) { return (unsigned)j < (unsigned)p.n; };
  auto idx_at = [&](long long s) { return s < end ? __ldg(idx + s) : -1; };
  auto consume = [&](const Frag<L, C, T>& f) {
    float kf[8];
    f.kc.to_f32(kf);
    float sp = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sp = fmaf(qv[e], kf[e], sp);
    for (int o = 1; o < G; o <<= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    const float sl = __shfl_sync(0xffffffffu, sp, src_lane);  // log2-scaled logit
    const bool raise = sl > mref + kLazy;
    if (__any_sync(0xffffffffu, raise)) {
      const float mnew = raise ? sl : mref;
      const float sc = raise ? fast_exp2(mref - mnew) : 1.f;
      z *= sc;
      const f32x2 sc2 = f2_pack(sc, sc);
#pragma unroll
      for (int t = 0; t < TPL; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = f2_mul(acc[t][e], sc2);
      mref = mnew;
    }
    const float pw = fast_exp2(sl - mref);
    z += pw;
    const f32x2 pw2 = f2_pack(pw, pw);
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      if (lane + 32 * t < NCH) {
        f32x2 hv[4];
        f.hc[t].to_f2(hv);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = f2_fma(pw2, hv[e], acc[t][e]);
      }
    }
  };

  // Two row buffers in ping-pong; neighbour indices are read four slots ahead
  // so the index load never sits on the path of a row gather.
  Frag<L, C, T> fa, fb;
  int j0 = idx_at(beg), j1 = idx_at(beg + 1), j2 = idx_at(beg + 2), j3 = idx_at(beg + 3);
  if (valid(j0)) fa.load(kp, hp, j0, lane, kch, hdk);
  for (long long s = beg; s < end; s += 2) {
    const int j4 = idx_at(s + 4), j5 = idx_at(s + 5);
    if (valid(j1)) fb.load(kp, hp, j1, lane, kch, hdk);
    if (valid(j0)) consume(fa);
    if (valid(j2)) fa.load(kp, hp, j2, lane, kch, hdk);
    if (valid(j1)) consume(fb);
    j0 = j2;
    j1 = j3;
    j2 = j4;
    j3 = j5;
  }

  const float inv = z > 0.f ? 1.f / z : 0.f;
  if constexpr (!FUSED) {
    float* o = p.out + (size_t)i * D * C;
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      const int q = lane + 32 * t;
      if (q < NCH) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) f2_unpack(acc[t][e], v[2 * e], v[2 * e + 1]);
        float4* dst = reinterpret_cast<float4*>(o + 8 * q);
        dst[0] = make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
        dst[1] = make_float4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
      }
    }
  } else {
    constexpr int WS = wig_size(L);
    float* mbuf = smem + wib * (D * C + WS);
    float* Dsm = mbuf + D * C;
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      const int q = lane + 32 * t;
      if (q < NCH) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) f2_unpack(acc[t][e], v[2 * e], v[2 * e + 1]);
#pragma unroll
        for (int e = 0; e < 8; ++e) mbuf[8 * q + e] = v[e] * inv;
      }
    }
    float Q[9];
    const float r = alignment_rotation(p.pos[3 * i], p.pos[3 * i + 1], p.pos[3 * i + 2], Q);
    float rpow[L + 1];
    rpow[0] = 1.f;
#pragma unroll
    for (int l = 1; l <= L; ++l) rpow[l] = rpow[l - 1] * r;
    wigner_build<L>(Q, Dsm, lane, 32, [] { __syncwarp(); });
    __syncwarp();
    float* o = p.out + (size_t)i * D * C;
#pragma unroll
    for (int c0 = 0; c0 < C; c0 += 32) {
      const int c = c0 + lane;
      if (c < C) {
        float xin[D];
#pragma unroll
        for (int d = 0; d < D; ++d) xin[d] = mbuf[d * C + c];
        eaas_channel<L>(xin, Dsm, rpow, p.tab,
                        [&](int pp) { return __ldg(p.w2 + pp * C + c); },
                        [&](int d, float v) { o[d * C + c] = v; });
      }
    }
  }
}

template <int L, int C, typename T, bool FUSED>
int launch_t(const AttnParams& p, cudaStream_t st) {
  constexpr int D = (L + 1) * (L + 1);
  const size_t shmem = FUSED ? size_t(kAttnWarps) * (D * C + wig_size(L)) * sizeof(float) : 0;
  auto kern = otf_attention_kernel<L, C, T, FUSED>;
  if (shmem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shmem)) !=
        cudaSuccess)
      return EGAT_ERR_CUDA;
  }
  const int grid = (p.n + kAttnWarps - 1) / kAttnWarps;
  kern<<<grid, kAttnWarps * 32, shmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

template <int L, typename T, bool FUSED>
int dispatch_c(const AttnParams& p, int C, cudaStream_t st) {
  switch (C) {
    case 16: return launch_t<L, 16, T, FUSED>(p, st);
    case 32: return launch_t<L, 32, T, FUSED>(p, st);
    case 64: return launch_t<L, 64, T, FUSED>(p, st);
    case 128: return launch_t<L, 128, T, FUSED>(p, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

template <typename T, bool FUSED>
int dispatch_l(const AttnParams& p, int L, int C, cudaStream_t st) {
  switch (L) {
    case 1: return dispatch_c<1, T, FUSED>(p, C, st);
    case 2: return dispatch_c<2, T, FUSED>(p, C, st);
    case 3: return dispatch_c<3, T, FUSED>(p, C, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_attention(const egat_shape& s, bool fused, const void* d_q, const void* d_k,
                     const void* d_hp, const int32_t* d_a, const int32_t* d_b,
                     const int32_t* d_order, const float* d_pos, const float* d_w2,
                     float* d_out, cudaStream_t st) {
  AttnParams p;
  p.q = d_q;
  p.k = d_k;
  p.hp = d_hp;
  p.nbr = d_a;
  p.cnt = d_b;
  p.order = d_order;
  p.out = d_out;
  p.pos = d_pos;
  p.w2 = d_w2;
  p.n = s.n;
  p.H = s.H;
  p.dk = s.dk;
  p.K = s.K;
  p.mode = s.graph_mode;
  p.n_edges = s.n_edges;
  p.qscale = float(1.4426950408889634 / std::sqrt(double(s.dk)));
  if (fused) p.tab = eaas_table(s.lmax);
  else memset(&p.tab, 0, sizeof(p.tab));
  const bool bf = s.dtype == EGAT_BF16;
  if (fused) {
    return bf ? dispatch_l<__nv_bfloat16, true>(p, s.lmax, s.C, st)
              : dispatch_l<float, true>(p, s.lmax, s.C, st);
  }
  return bf ? dispatch_l<__nv_bfloat16, false>(p, s.lmax, s.C, st)
            : dispatch_l<float, false>(p, s.lmax, s.C, st);
}

}  // namespace egat
