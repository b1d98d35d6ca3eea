// Invariant query/key projection: q_i, k_i from the degree-0 channels of h_i.
//
// "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
// Memory" §2.2 (Eq. 6): queries and keys are SO(3)-invariant scalar
// projections of the node features; the equivariant geometry travels only
// along the value path.  Reading: a linear map without bias of the C
// degree-0 channels (component 0 of each atom's [D][C] row, the invariant
// scalars) to every head,
//     q[i][h*dk + d] = sum_c h[i][0][c] wq[c][h*dk + d],   k likewise with wk.
//
// This is a dense contraction, [n x C] . [C x H*dk] twice, so the bf16
// shapes with C = 128 and H*dk = 256 run on tensor cores:
//  * a persistent CTA holds one weight matrix (wq or wk, by CTA parity) in
//    shared memory as a bf16 pair hi + lo (hi = bf16(w), lo = bf16(w - hi)),
//    transposed [H*dk][C] so that ldmatrix yields mma B fragments; the pair
//    carries the float32 weights to about 2^-17, and h is exactly bf16;
//  * tiles of 64 atoms: one thread issues one 256-byte bulk copy per atom
//    (the degree-0 slice of its row; cp.async.bulk, no multicast) into a
//    ring of four row-padded A tiles, each completing its own mbarrier, so
//    three tiles are in flight while one is multiplied; every wait is bounded;
//  * 16 warps, each 32 atoms x 32 output columns: per 16-channel k-step two
//    A fragments (ldmatrix.x4), two B fragment pairs for hi and lo, and 16
//    mma.sync m16n8k16 (bf16 in, float32 accumulation);
//  * the accumulators are rounded once to the storage type and stored.
// It moves n * (C + 2 * H*dk) * 2 bytes (degree-0 slices in, q and k out):
// an HBM-bound contraction (K = C = 128 gives 64 FLOP per stored byte of
// output at most), so the kernel is measured against HBM bandwidth.
//
// Other shapes (float32 storage, other C or H*dk) take a plain kernel: a CTA
// stages the degree-0 channels of 8 atoms and each thread forms output
// columns as float32 dot products over C, reading the weights from L2.
#include <cuda_bf16.h>

#include "egat_async.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kPC = 128;          // channels (the contraction length)
constexpr int kPN = 256;          // H * dk outputs per matrix
constexpr int kPM = 64;           // atoms per tile
constexpr int kPRow = kPC * 2 + 16;   // padded bf16 row (272 B): ldmatrix phases hit distinct banks
constexpr int kPWarps = 16;
constexpr int kPBuf = 4;              // A tiles in the ring

struct ProjSmem {
  static constexpr size_t whi = 0;                                   // [kPN][kPRow]
  static constexpr size_t wlo = whi + size_t(kPN) * kPRow;           // [kPN][kPRow]
  static constexpr size_t a = wlo + size_t(kPN) * kPRow;             // [kPBuf][kPM][kPRow]
  static constexpr size_t bars = a + size_t(kPBuf) * kPM * kPRow;    // [kPBuf] mbarriers + abort flag
  static constexpr size_t total = bars + kPBuf * 8 + 16;
  static_assert(kPRow % 16 == 0 && a % 16 == 0 && bars % 8 == 0, "bulk-copy alignment");
};

struct ProjParams {
  const __nv_bfloat16* h;
  const float* w[2];      // wq, wk  [kPC][kPN]
  __nv_bfloat16* out[2];  // q, k    [n][kPN]
  long long row_elems;    // D * C: elements per atom row of h
  int n;
  int tiles;
};

__device__ __forceinline__ void pj_ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void pj_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kPWarps * 32, 1) qk_projection_tc_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* whi = smem + ProjSmem::whi;
  unsigned char* wlo = smem + ProjSmem::wlo;
  unsigned char* abuf = smem + ProjSmem::a;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + ProjSmem::bars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kPBuf);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sel = blockIdx.x & 1;            // 0: q from wq, 1: k from wk
  const int slot = blockIdx.x >> 1;
  const int stride = gridDim.x >> 1;
  if (slot >= p.tiles) return;               // whole CTA

  if (tid == 0) {
    for (int b = 0; b < kPBuf; ++b) mbar_init(smem_u32(bar + b), 1);
    mbar_fence_init();
    *abort_flag = 0;
  }
  // weights: float32 [c][col] -> transposed bf16 hi/lo [col][c], stored as
  // (c, c + 1) pairs.  A warp converts a block of 8 columns x 4 channel
  // pairs: lane -> column 8 cb + (lane & 7), pair 4 pb + (lane >> 3).  With
  // the 68-word row pitch its 32 four-byte stores hit 32 distinct banks, and
  // each load instruction reads 8 full 32-byte sectors.  Every load of the
  // thread is issued before the first conversion.
  const float* w = p.w[sel];
  constexpr int kPer = (kPC / 2) * kPN / (kPWarps * 32);   // pairs per thread
  static_assert((kPC / 2) * kPN % (kPWarps * 32 * 32) == 0 && kPN % 8 == 0, "weight blocks");
  float x0[kPer], x1[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int blk = i * kPWarps + warp;
    const int col = (blk % (kPN / 8)) * 8 + (lane & 7);
    const int c = 2 * ((blk / (kPN / 8)) * 4 + (lane >> 3));
    x0[i] = __ldg(w + c * kPN + col);
    x1[i] = __ldg(w + (c + 1) * kPN + col);
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int blk = i * kPWarps + warp;
    const int col = (blk % (kPN / 8)) * 8 + (lane & 7);
    const int c = 2 * ((blk / (kPN / 8)) * 4 + (lane >> 3));
    const __nv_bfloat162 hi = __floats2bfloat162_rn(x0[i], x1[i]);
    const __nv_bfloat162 lo =
        __floats2bfloat162_rn(x0[i] - __low2float(hi), x1[i] - __high2float(hi));
    *reinterpret_cast<__nv_bfloat162*>(whi + size_t(col) * kPRow + c * 2) = hi;
    *reinterpret_cast<__nv_bfloat162*>(wlo + size_t(col) * kPRow + c * 2) = lo;
  }
  __syncthreads();

  const char* hb = reinterpret_cast<const char*>(p.h);
  const long long row_bytes = p.row_elems * 2;
  // thread 0: the degree-0 slices (first 256 bytes of each row) of tile tl
  auto issue = [&](int tl, int b) {
    const int a0 = tl * kPM;
    const int valid = p.n - a0 < kPM ? p.n - a0 : kPM;
    const uint32_t bb = smem_u32(bar + b);
    mbar_arrive_expect_tx(bb, uint32_t(valid) * (kPC * 2));
    for (int r = 0; r < valid; ++r)
      bulk_g2s(smem_u32(abuf + (size_t(b) * kPM + r) * kPRow), hb + (long long)(a0 + r) * row_bytes,
               kPC * 2, bb);
  };
  // the ring starts with the CTA's first kPBuf - 1 tiles in flight
  if (tid == 0)
    for (int q = 0; q < kPBuf - 1 && slot + q * stride < p.tiles; ++q) issue(slot + q * stride, q);

  const int g = lane >> 2, t = lane & 3;
  const int m0 = (warp & 1) * 32;            // this warp's first atom of the tile
  const int n0 = (warp >> 1) * 32;           // this warp's first output column
  __nv_bfloat16* out = p.out[sel];
  int j = 0;
  for (int tile = slot; tile < p.tiles; tile += stride, ++j) {
    const int b = j % kPBuf;
    bounded_wait(smem_u32(bar + b), uint32_t(j / kPBuf) & 1u, kWaitPolls, abort_flag);
    // the tile kPBuf - 1 ahead into the buffer tile j - 1 used (it ended
    // with a barrier)
    const int ahead = tile + (kPBuf - 1) * stride;
    if (tid == 0 && ahead < p.tiles) issue(ahead, (j + kPBuf - 1) % kPBuf);
    float acc[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    const uint32_t a_base = smem_u32(abuf + size_t(b) * kPM * kPRow);
    const int arow = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int brow = (lane & 7) + 8 * (lane >> 4);
    const int bhalf = (lane >> 3) & 1;
#pragma unroll 2
    for (int kk = 0; kk < kPC / 16; ++kk) {
      uint32_t af[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
        pj_ldsm_x4(af[mt], a_base + (m0 + mt * 16 + arow) * kPRow + kk * 32 + (lane >> 4) * 16);
#pragma unroll
      for (int np = 0; np < 2; ++np) {       // pairs of n8 tiles
        uint32_t bh[4], bl[4];
        const uint32_t off = (n0 + np * 16 + brow) * kPRow + kk * 32 + bhalf * 16;
        pj_ldsm_x4(bh, smem_u32(whi) + off);
        pj_ldsm_x4(bl, smem_u32(wlo) + off);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          pj_mma(acc[mt][2 * np], af[mt], bh[0], bh[1]);
          pj_mma(acc[mt][2 * np + 1], af[mt], bh[2], bh[3]);
          pj_mma(acc[mt][2 * np], af[mt], bl[0], bl[1]);
          pj_mma(acc[mt][2 * np + 1], af[mt], bl[2], bl[3]);
        }
      }
    }
    // rows g and g+8 of each m tile, columns 2t, 2t+1 of each n tile
    const int a0 = tile * kPM + m0;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int atom = a0 + mt * 16 + g + 8 * half;
        if (atom < p.n) {
          __nv_bfloat16* o = out + (long long)atom * kPN + n0 + 2 * t;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
            *reinterpret_cast<__nv_bfloat162*>(o + nt * 8) =
                __floats2bfloat162_rn(acc[mt][nt][2 * half], acc[mt][nt][2 * half + 1]);
        }
      }
    __syncthreads();   // buffer b is refilled by a later iteration's issue
  }
  if (*abort_flag && tid == 0) {
    // a wait gave up: give each buffer's last issued phase a short, bounded
    // chance to complete before the CTA's shared memory is released (tile
    // sequence numbers up to j + kPBuf - 2 may have been issued)
    volatile int none = 0;
    for (int b = 0; b < kPBuf; ++b) {
      int last = -1;
      for (int q = 0; q < j + kPBuf - 1; ++q)
        if (q % kPBuf == b && slot + q * stride < p.tiles) last = q;
      if (last >= 0)
        bounded_wait(smem_u32(bar + b), uint32_t(last / kPBuf) & 1u, kDrainPolls, &none);
    }
  }
}

// Plain path: 8 atoms per CTA, their degree-0 channels staged as float32;
// thread c0 forms output columns c0, c0 + blockDim, ... of q then k.
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kGenAtoms = 8;
template <typename T>
__global__ void __launch_bounds__(256) qk_projection_kernel(const T* __restrict__ h, const float* __restrict__ wq,
                                                            const float* __restrict__ wk, T* __restrict__ q,
                                                            T* __restrict__ k, long long row_elems, int n,
                                                            int C, int HD) {
  extern __shared__ float h0[];   // [kGenAtoms][C]
  const int a0 = blockIdx.x * kGenAtoms;
  const int na = n - a0 < kGenAtoms ? n - a0 : kGenAtoms;
  for (int e = threadIdx.x; e < na * C; e += blockDim.x) {
    const int a = e / C, c = e % C;
    h0[e] = to_f<T>(h[(long long)(a0 + a) * row_elems + c]);
  }
  __syncthreads();
  for (int col = threadIdx.x; col < 2 * HD; col += blockDim.x) {
    const float* w = col < HD ? wq + col : wk + (col - HD);
    float acc[kGenAtoms];
#pragma unroll
    for (int a = 0; a < kGenAtoms; ++a) acc[a] = 0.f;
    for (int c = 0; c < C; ++c) {
      const float wc = __ldg(w + (long long)c * HD);
#pragma unroll
      for (int a = 0; a < kGenAtoms; ++a) acc[a] = fmaf(h0[a * C + c], wc, acc[a]);
    }
    T* o = col < HD ? q + col : k + (col - HD);
    for (int a = 0; a < na; ++a) o[(long long)(a0 + a) * HD] = from_f<T>(acc[a]);
  }
}

}  // namespace

bool projection_tc_supported(const egat_shape& s) {
  return s.dtype == EGAT_BF16 && s.C == kPC && s.H * s.dk == kPN;
}

int launch_qk_projection(const egat_shape& s, const void* d_h, const float* d_wq, const float* d_wk,
                         void* d_q, void* d_k, cudaStream_t st) {
  const long long row_elems = (long long)(s.lmax + 1) * (s.lmax + 1) * s.C;
  const int HD = s.H * s.dk;
  if (projection_tc_supported(s)) {
    ProjParams p;
    p.h = static_cast<const __nv_bfloat16*>(d_h);
    p.w[0] = d_wq;
    p.w[1] = d_wk;
    p.out[0] = static_cast<__nv_bfloat16*>(d_q);
    p.out[1] = static_cast<__nv_bfloat16*>(d_k);
    p.row_elems = row_elems;
    p.n = s.n;
    p.tiles = (s.n + kPM - 1) / kPM;
    const size_t shmem = ProjSmem::total;
    if (cudaFuncSetAttribute(qk_projection_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(shmem)) != cudaSuccess)
      return EGAT_ERR_CUDA;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one CTA per SM, an even count: CTA pairs share atom tiles, one for q, one for k
    const int pairs = p.tiles < sms / 2 ? p.tiles : sms / 2;
    qk_projection_tc_kernel<<<2 * (pairs > 0 ? pairs : 1), kPWarps * 32, shmem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
  }
  const int blocks = (s.n + kGenAtoms - 1) / kGenAtoms;
  const size_t shmem = size_t(kGenAtoms) * s.C * sizeof(float);
  if (s.dtype == EGAT_BF16)
    qk_projection_kernel<__nv_bfloat16><<<blocks, 256, shmem, st>>>(
        static_cast<const __nv_bfloat16*>(d_h), d_wq, d_wk, static_cast<__nv_bfloat16*>(d_q),
        static_cast<__nv_bfloat16*>(d_k), row_elems, s.n, s.C, HD);
  else
    qk_projection_kernel<float><<<blocks, 256, shmem, st>>>(
        static_cast<const float*>(d_h), d_wq, d_wk, static_cast<float*>(d_q),
        static_cast<float*>(d_k), row_elems, s.n, s.C, HD);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

int take_wait_timeouts_projection(cudaStream_t st, unsigned int* count) {
  return take_unit_wait_timeouts(st, count) == 0 ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
