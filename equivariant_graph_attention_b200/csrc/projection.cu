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
// shapes with C = 128 and H*dk = 256 run on the fifth-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory):
//  * a persistent CTA per SM holds one weight matrix (wq or wk, by CTA
//    parity) in shared memory as a bf16 pair hi + lo (hi = bf16(w),
//    lo = bf16(w - hi)), transposed to [H*dk][C]; the pair carries the
//    float32 weights to about 2^-17, and h is exactly bf16.  The float32
//    matrix arrives in two 64 KB bulk copies (cp.async.bulk, no multicast)
//    and is converted from shared memory;
//  * per 128-atom tile the degree-0 slices (256 bytes per atom) arrive by two
//    TMA tensor copies (cp.async.bulk.tensor.2d, 64 channels x 128 atoms
//    each, 128-byte swizzle, rows past n zero-filled; no multicast) on the
//    buffer's mbarrier, two tiles in flight, and one thread issues
//    sixteen 128 x 256 x 16 products (h W_hi and h W_lo per 16-channel step)
//    into one of two 256-column float32 accumulators in tensor memory,
//    completing that accumulator's mbarrier; tile j + 1's products run while
//    tile j is read back;
//  * eight warps read the accumulator back (tcgen05.ld), round once to the
//    storage type and store through shared memory, 64 contiguous bytes of a
//    row per four lanes.  Every wait is bounded.
// It moves n * (C + 2 * H*dk) * 2 bytes (degree-0 slices in, q and k out):
// K = C = 128 gives at most 64 FLOP per stored byte of output, so the
// kernel is measured against HBM bandwidth.
//
// Other shapes (float32 storage, other C or H*dk) take a plain kernel: a CTA
// stages the degree-0 channels of 8 atoms and each thread forms output
// columns as float32 dot products over C, reading the weights from L2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "egat_async.cuh"
#include "egat_host.h"

namespace egat {
namespace {

struct ProjParams {
  CUtensorMap amap;       // h's degree-0 slices as a [n][C] bf16 matrix (row pitch D * C * 2 bytes)
  const float* w[2];      // wq, wk  [C][H*dk]
  __nv_bfloat16* out[2];  // q, k    [n][H*dk]
  int n;
  int tiles;              // 128-atom tiles
};

// ---------------------------------------------------------------- tcgen05 path
// One CTA per SM holds one weight matrix (wq or wk, by CTA parity) as bf16
// hi and lo tiles and takes 128-atom tiles:
//  * A (the tile's degree-0 slices, 128 x 128 bf16) arrives by two TMA
//    tensor copies on the buffer's mbarrier, two tiles in flight (a ragged
//    tile's missing rows arrive as zeros);
//  * one thread issues the tile's 16 tcgen05.mma (M = 128, N = 256, K = 16:
//    eight k-steps, each against the hi and the lo tile), accumulating
//    h W_hi + h W_lo in float32 into one of two 256-column accumulators in
//    tensor memory, and commits them to that accumulator's mbarrier;
//  * eight warps read the accumulator back (tcgen05.ld, each warp its
//    32-lane quarter and half of the columns), round to bf16 and store.
// Shared-memory operands, both K-major: A (the atoms' channels) in the
// 128-byte-swizzled layout the tensor copy writes (per 64-channel half, 128
// rows of 128 bytes, 16-byte chunks permuted by row % 8; 8-row groups 1 KB
// apart; a 16-channel k-step starts 32 bytes further along the row); B (the
// weights, written by this kernel) in the no-swizzle canonical layout: 8-row
// x 16-byte core matrices of 128 contiguous bytes, 8-row groups 128 bytes
// apart (SBO), the two 8-channel halves of a k-step one channel chunk apart
// (LBO).
constexpr int kUM = 128;                 // atoms per tile (M)
constexpr int kUN = 256;                 // outputs per matrix (N)
constexpr int kUK = 128;                 // channels (K)
constexpr int kUWarps = 8;
constexpr int kUHalfA = kUM * 128;       // bytes per 64-channel half of an A tile (swizzled rows)
constexpr int kUChunkB = kUN * 16;       // bytes per 8-channel chunk of a B tile
constexpr int kUCols = 512;              // tensor-memory columns: two float32 accumulators of N = 256
constexpr int kUStageRow = 80;           // a staged 64-byte output row segment, padded (bank spread)

struct UmmaSmem {
  static constexpr size_t bhi = 0;                                      // [16][32][8][16 B]
  static constexpr size_t blo = bhi + size_t(kUK / 8) * kUChunkB;
  static constexpr size_t a = blo + size_t(kUK / 8) * kUChunkB;         // [2][2 halves][128][128 B]
  static constexpr size_t stage = a + 2 * size_t(2) * kUHalfA;          // [8 warps][32 rows][80 B]
  static constexpr size_t bars = stage + size_t(kUWarps) * 32 * kUStageRow;  // products [2], A [2], weights
  static constexpr size_t tslot = bars + 40;                             // tensor-memory address
  static constexpr size_t flag = tslot + 4;                              // abort flag
  static constexpr size_t total = flag + 4 + 16;
  static_assert(a % 1024 == 0 && kUHalfA % 1024 == 0 && bars % 8 == 0, "operand alignment");
};

// Shared-memory matrix descriptor: start, leading and stride byte offsets
// (16-byte units), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}
// the same for a 128-byte-swizzled K-major operand (layout type 2): 8-row
// groups 1 KB apart, the leading offset unused (16 bytes)
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return umma_desc(saddr, 16, 1024) | (uint64_t(2) << 61);
}
// 2-D tensor copy of box {x, y} of the map into shared memory, completing bar
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// Instruction descriptor, kind::f16: float32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kUIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kUN >> 3) << 17) |
                             (uint32_t(kUM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kUIdesc), "r"(uint32_t(accumulate))
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// 32 consecutive float32 columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__global__ void __launch_bounds__(kUWarps * 32, 1) qk_projection_umma_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* bhi = smem + UmmaSmem::bhi;
  unsigned char* blo = smem + UmmaSmem::blo;
  unsigned char* abuf = smem + UmmaSmem::a;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + UmmaSmem::bars);        // [2] products per accumulator
  uint64_t* abar = bar + 2;                                                   // [2] an A buffer's copies
  uint64_t* wbar = bar + 4;                                                   // a weight half
  unsigned char* stage = smem + UmmaSmem::stage;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + UmmaSmem::tslot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + UmmaSmem::flag);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sel = blockIdx.x & 1;            // 0: q from wq, 1: k from wk
  const int slot = blockIdx.x >> 1;
  const int stride = gridDim.x >> 1;
  if (slot >= p.tiles) return;               // whole CTA

  if (tid == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(smem_u32(bar + b), 1);
    mbar_fence_init();
    *abort_flag = 0;
  }
  if (warp == 0) {
    // 512 columns of tensor memory, two accumulators (one CTA per SM: the
    // shared memory fills it, so the allocation never waits on another CTA)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tslot)),
                 "r"(kUCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }

  // thread 0: tile tl's degree-0 slices into A buffer b, two 64-channel
  // halves of 128 rows (rows past n arrive as zeros)
  int loaded = 0;   // tiles whose copies were issued (this CTA's sequence numbers)
  auto load_tile = [&](int jj, int b) {
    const int tl = slot + jj * stride;
    if (tid == 0 && tl < p.tiles) {
      const uint32_t ab = smem_u32(abar + b);
      const uint32_t dst = smem_u32(abuf + size_t(b) * 2 * kUHalfA);
      mbar_arrive_expect_tx(ab, 2u * kUHalfA);
      tma_load_2d(dst, &p.amap, 0, tl * kUM, ab);
      tma_load_2d(dst + kUHalfA, &p.amap, 64, tl * kUM, ab);
    }
    if (tl < p.tiles) loaded = jj + 1;
  };
  // weights: float32 [k][n] -> bf16 hi / lo at (k / 8) * kUChunkB +
  // (n / 8) * 128 + (n % 8) * 16 + (k % 8) * 2, stored as (k, k + 1) pairs.
  // A warp converts 8 columns x 4 channel pairs per step: lane -> column
  // 8 nb + (lane & 7), pair 4 kb + (lane >> 3); its 32 four-byte stores hit
  // 32 distinct banks.
  auto put = [&](int k, int n, float x0, float x1) {
    const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - __low2float(hi), x1 - __high2float(hi));
    const size_t off = size_t(k >> 3) * kUChunkB + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat162*>(bhi + off) = hi;
    *reinterpret_cast<__nv_bfloat162*>(blo + off) = lo;
  };
  const float* w = p.w[sel];
  const bool staged = (reinterpret_cast<uintptr_t>(w) & 15u) == 0;
  if (staged) {
    // 16-byte aligned weights arrive as two bulk copies of 64 rows (64 KB of
    // float32 each) into the A buffers, which are free until the first tile
    const float* stage = reinterpret_cast<const float*>(abuf);
    constexpr int kRows = kUK / 2;
    static_assert(size_t(kRows) * kUN * 4 <= 2 * size_t(2) * kUHalfA, "a weight half fits the A buffers");
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      if (tid == 0) {
        mbar_arrive_expect_tx(smem_u32(wbar), uint32_t(kRows) * kUN * 4);
        bulk_g2s(smem_u32(abuf), w + size_t(half) * kRows * kUN, uint32_t(kRows) * kUN * 4, smem_u32(wbar));
      }
      bounded_wait(smem_u32(wbar), uint32_t(half), kWaitPolls, abort_flag);
#pragma unroll 4
      for (int blk = warp; blk < (kUN / 8) * (kRows / 8); blk += kUWarps) {
        const int n = (blk % (kUN / 8)) * 8 + (lane & 7);
        const int k = 2 * ((blk / (kUN / 8)) * 4 + (lane >> 3));   // row within the half
        put(half * kRows + k, n, stage[k * kUN + n], stage[(k + 1) * kUN + n]);
      }
      __syncthreads();   // the half is consumed before the buffers are refilled
    }
  } else {
    // other weights: every thread loads its pairs straight from global memory
    constexpr int kBlocks = (kUN / 8) * (kUK / 8);   // 8 x 8 blocks: 512
    constexpr int kBatch = 16;                       // blocks in flight per warp
#pragma unroll 1
    for (int b0 = warp * kBatch; b0 < kBlocks; b0 += kUWarps * kBatch) {
      float x0[kBatch], x1[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int blk = b0 + i;
        const int n = (blk % (kUN / 8)) * 8 + (lane & 7);
        const int k = 2 * ((blk / (kUN / 8)) * 4 + (lane >> 3));
        x0[i] = __ldg(w + k * kUN + n);
        x1[i] = __ldg(w + (k + 1) * kUN + n);
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int blk = b0 + i;
        put(2 * ((blk / (kUN / 8)) * 4 + (lane >> 3)), (blk % (kUN / 8)) * 8 + (lane & 7), x0[i], x1[i]);
      }
    }
  }
  fence_proxy_async_smem();   // the staged weights were read before the tensor copies overwrite them
  __syncthreads();
  load_tile(0, 0);
  load_tile(1, 1);
  fence_proxy_async_smem();   // the weight tiles are read by the tensor core
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = *tslot;

  __nv_bfloat16* out = p.out[sel];
  const int quarter = warp & 3, colh = warp >> 2;   // TMEM lanes 32 quarter.., columns 128 colh..
  const int J = (p.tiles - slot + stride - 1) / stride;   // this CTA's tiles
  // tile jj's products from A buffer jj % 2 into accumulator jj % 2 (columns
  // 256 (jj % 2) ..), completing mbarrier jj % 2; every thread takes part
  // (the wait for the tile's copies and the barrier before the issue)
  auto issue = [&](int jj) {
    tmem_fence_before();         // the accumulator's previous reads are done
    __syncthreads();
    if (tid == 0) {
      const int b = jj & 1;
      bounded_wait(smem_u32(abar + b), uint32_t(jj >> 1) & 1u, kWaitPolls, abort_flag);   // the tile's copies
      tmem_fence_after();
      const uint32_t acc = tmem + uint32_t(b * kUN);
      const uint32_t a0 = smem_u32(abuf + size_t(b) * 2 * kUHalfA);
      const uint32_t h0 = smem_u32(bhi), l0 = smem_u32(blo);
#pragma unroll
      for (int s = 0; s < kUK / 16; ++s) {
        const uint64_t ad = umma_desc_sw128(a0 + (s >> 2) * kUHalfA + (s & 3) * 32);
        umma_bf16(acc, ad, umma_desc(h0 + 2 * s * kUChunkB, kUChunkB, 128), s > 0);
        umma_bf16(acc, ad, umma_desc(l0 + 2 * s * kUChunkB, kUChunkB, 128), true);
      }
      umma_commit(smem_u32(bar + b));
    }
  };
  unsigned char* wst = stage + size_t(warp) * 32 * kUStageRow;   // this warp's staging rows
  bool ok = true;
  int issued = 0, j = 0;
  if (J > 0) {
    issue(0);
    issued = 1;
  }
  for (; j < J; ++j) {
    const int tile = slot + j * stride;
    const int b = j & 1;
    // the next tile's products run while this one is read back
    if (j + 1 < J) {
      issue(j + 1);
      issued = j + 2;
    }
    // every thread leaves together if the commit never arrives
    ok = __syncthreads_and(bounded_wait(smem_u32(bar + b), uint32_t(j >> 1) & 1u, kWaitPolls, abort_flag));
    if (!ok) break;
    tmem_fence_after();
    // A buffer b is free: the tile two ahead goes there
    load_tile(j + 2, b);
    // read back 32 columns at a time: each lane its atom's row segment, as
    // bf16 through the warp's staging rows, then stored as 8 rows x 64
    // contiguous bytes per instruction
    const long long row0 = (long long)tile * kUM + quarter * 32;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + uint32_t(b * kUN) + (uint32_t(quarter * 32) << 16) + uint32_t(colh * 128 + c * 32), r);
      tmem_ld_wait();
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t wv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(r[8 * v + 2 * e]),
                                                          __uint_as_float(r[8 * v + 2 * e + 1]));
          wv[e] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(wst + lane * kUStageRow + v * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = i * 8 + (lane >> 2), seg = lane & 3;
        const long long atom = row0 + rr;
        const uint4 v4 = *reinterpret_cast<const uint4*>(wst + rr * kUStageRow + seg * 16);
        if (atom < p.n)
          *reinterpret_cast<uint4*>(out + atom * kUN + colh * 128 + c * 32 + seg * 8) = v4;
      }
      __syncwarp();   // the staging rows are rewritten by the next column block
    }
  }
  if (*abort_flag && tid == 0) {
    // a wait gave up: a short, bounded chance for the products, tile copies
    // and weight copies in flight to finish before tensor and shared memory
    // are released
    volatile int none = 0;
    for (int bb = 0; bb < 2; ++bb) {
      int last = issued - 1;
      while (last >= 0 && (last & 1) != bb) --last;
      if (last >= 0) bounded_wait(smem_u32(bar + bb), uint32_t(last >> 1) & 1u, kDrainPolls, &none);
      last = loaded - 1;
      while (last >= 0 && (last & 1) != bb) --last;
      if (last >= 0) bounded_wait(smem_u32(abar + bb), uint32_t(last >> 1) & 1u, kDrainPolls, &none);
    }
    if (staged)
      for (int half = 0; half < 2; ++half) bounded_wait(smem_u32(wbar), uint32_t(half), kDrainPolls, &none);
  }
  tmem_fence_before();
  __syncthreads();
  if (warp == 0) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kUCols) : "memory");
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

// The tensor map of h's degree-0 slices: a [n][C] bf16 matrix whose rows lie
// D * C * 2 bytes apart, read in boxes of 64 channels x 128 atoms with the
// 128-byte swizzle (the A operand layout of qk_projection_umma_kernel).  The
// encoder comes from the driver through the runtime's entry-point query.
int encode_degree0_map(CUtensorMap* map, const void* d_h, int n, long long row_elems) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return -1;
  const cuuint64_t dims[2] = {cuuint64_t(kUK), cuuint64_t(n)};
  const cuuint64_t strides[1] = {cuuint64_t(row_elems) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(kUM)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(d_h), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

bool projection_tc_supported(const egat_shape& s) {
  return s.dtype == EGAT_BF16 && s.C == kUK && s.H * s.dk == kUN;
}

int launch_qk_projection(const egat_shape& s, const void* d_h, const float* d_wq, const float* d_wk,
                         void* d_q, void* d_k, cudaStream_t st) {
  const long long row_elems = (long long)(s.lmax + 1) * (s.lmax + 1) * s.C;
  const int HD = s.H * s.dk;
  // the tensor-core kernel stores 16-byte row segments of q and k
  const bool out16 = ((reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_k)) & 15u) == 0;
  if (projection_tc_supported(s) && out16) {
    ProjParams p;
    if (encode_degree0_map(&p.amap, d_h, s.n, row_elems) != 0) return EGAT_ERR_CUDA;
    p.w[0] = d_wq;
    p.w[1] = d_wk;
    p.out[0] = static_cast<__nv_bfloat16*>(d_q);
    p.out[1] = static_cast<__nv_bfloat16*>(d_k);
    p.n = s.n;
    p.tiles = (s.n + kUM - 1) / kUM;
    const size_t shmem = UmmaSmem::total;
    if (cudaFuncSetAttribute(qk_projection_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(shmem)) != cudaSuccess)
      return EGAT_ERR_CUDA;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one CTA per SM, an even count: CTA pairs share atom tiles, one for q, one for k
    const int pairs = p.tiles < sms / 2 ? p.tiles : sms / 2;
    qk_projection_umma_kernel<<<2 * (pairs > 0 ? pairs : 1), kUWarps * 32, shmem, st>>>(p);
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
