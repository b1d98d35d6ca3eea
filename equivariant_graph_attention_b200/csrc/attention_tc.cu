// Step 3 (+4) on tensor cores: tiles of kTileM targets share one pass over
// the union of their neighbours.
//
// What is computed is exactly the on-the-fly attention of
// "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.1-§3.2 and
// "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
// Memory" §2.2: per target and head a softmax of q_i.k_j/sqrt(dk) over the
// target's own neighbours, m_i = sum_j alpha_ij h'_j accumulated on chip with
// an online softmax, and (fused) ^h_i = m_i (x) R(r_i) by EAAS.  Nothing per
// edge reaches memory.
//
// How it maps to B200: a tile of 16 spatially adjacent targets (consecutive
// in the cell order) reads each row of the union of their neighbour lists
// once.  A persistent CTA per SM, one warp per head; per tile:
//  * the tile's union indices and membership mask (from the plan) go to
//    shared memory, and so does its record: the 16 target ids, |r|^l and the
//    Wigner-D matrices of their alignment rotations, built once per atom by
//    the plan, so nothing is rebuilt here;
//  * the union streams through shared memory in stages of RS rows, STAGES
//    stages in flight: one thread per row issues its value row and key row as
//    two bulk copies (cp.async.bulk, the TMA engine's 1-D form, no multicast)
//    that complete the stage buffer's mbarrier by their byte count; rows are
//    padded by 16 bytes so ldmatrix phases hit distinct banks.  Every wait on
//    an mbarrier is bounded (bounded_wait): a wait that gives up is counted
//    for egat_take_device_status and the CTA stops waiting, so no launch can
//    hang;
//  * per 16 union atoms and head, S = Q_h K_h^T with two mma.sync m16n8k16
//    (bf16 in, f32 out), the key fragments by one ldmatrix.x4;
//  * the plan's membership bits mask S to each target's own neighbours; the
//    online softmax keeps a per-row reference maximum raised lazily (only by
//    more than 2^8), tested once per stage, so z and the accumulators share
//    one reference; z is the mma of P with an all-ones fragment — the row
//    sums of exactly the bf16 weights that enter P V;
//  * the probabilities become the bf16 A fragment directly (the S fragment
//    layout of two n8 tiles is the A layout of one k16 step) and P V_h runs
//    as one mma.sync per component of the head's 8 channels, the value
//    fragments by ldmatrix.trans from the staged rows.
// The accumulator fragment of a lane holds, for targets g and g+8 and
// channels 2t, 2t+1 of its head, every component d — exactly what the
// per-channel EAAS epilogue needs, so the target coupling runs from registers.
#include <cfloat>

#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kRowPad = 16;   // bytes of padding per staged row
// stage mbarriers (up to 3) and the abort flag, after 16-byte alignment
constexpr size_t kBarBytes = 16 + 8 * 3 + 8;

struct TcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* hp;
  PlanView plan;
  const int32_t* order;
  float* out;
  const float* pos;
  const float* w2;
  int n;
  float qscale;   // log2(e) / sqrt(dk)
  EaasTable tab;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// mbarrier and bulk-copy (TMA engine, no multicast) helpers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Waits that gave up since the last egat_take_device_status (all launches on
// this device).
__device__ unsigned int g_wait_timeouts;
// Polls before a wait gives up.  try_wait suspends the thread for at most a
// hardware-defined interval per poll, so this bounds a wait to about a
// second; a stage's copies normally land within microseconds.
constexpr int kWaitPolls = 1 << 20;
constexpr int kDrainPolls = 1 << 14;

// Wait until the phase of parity `parity` of the mbarrier at `bar` has
// completed, polling at most `polls` times.  On giving up: count it, set the
// CTA's abort flag and return false; once the flag is set, waits return at
// once, so a CTA whose copies never land finishes its loop (with meaningless
// results, reported by egat_take_device_status) instead of hanging.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, int polls,
                                             volatile int* abort_flag) {
  if (*abort_flag) return false;
  for (int i = 0; i < polls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  atomicAdd(&g_wait_timeouts, 1u);
  *abort_flag = 1;
  return false;
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
// D += A B for one m16n8k16 tile, bf16 inputs, f32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A pipeline stage holds KS k-steps (KS * kTileK union rows): one barrier per
// stage; STAGES stages are in flight.
template <int L>
struct TcShape {
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int KS = L >= 3 ? 1 : 2;
  static constexpr int STAGES = L >= 3 ? 2 : (L == 2 ? 2 : 3);
  static constexpr int RS = KS * kTileK;   // rows per stage
};

// staging buffers, then the tile's Wigner-D / |r|^l / targets, then the tile's
// union indices [cap] and membership mask [kTileM][cap / 32]
template <int L, int H>
constexpr size_t tc_smem_fixed() {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int C = 8 * H;
  constexpr int VSTR = D * C * 2 + kRowPad;
  constexpr int KSTR = H * 16 * 2 + kRowPad;
  return size_t(TcShape<L>::STAGES) * TcShape<L>::RS * (VSTR + KSTR) +
         size_t(kTileM) * (wig_size(L) + L + 1) * sizeof(float) + kTileM * sizeof(int);
}
// mask rows are padded by one word so the 8 rows a warp reads sit in distinct banks
// fused kernels keep the target-coupling weights [P][C] in shared memory
template <int L, int H>
constexpr size_t tc_smem_w2() {
  return size_t(num_paths(L)) * 8 * H * sizeof(float);
}
inline size_t tc_smem_plan(int cap) {
  return size_t(cap) * sizeof(int) + size_t(kTileM) * (cap / 32 + 1) * sizeof(uint32_t);
}

template <int L, int H, bool FUSED>
__global__ void __launch_bounds__(H * 32, 1)
otf_attention_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int D = (L + 1) * (L + 1);
  constexpr int C = 8 * H;
  constexpr int ROW = D * C * 2;                  // value row bytes
  constexpr int VSTR = ROW + kRowPad;
  constexpr int KROW = H * 16 * 2;                // key row bytes (dk = 16)
  constexpr int KSTR = KROW + kRowPad;
  constexpr int STAGES = TcShape<L>::STAGES;
  constexpr int KS = TcShape<L>::KS;
  constexpr int RS = TcShape<L>::RS;
  constexpr int WS = wig_size(L);
  constexpr int NTHR = H * 32;
  constexpr int VCH = ROW / 16, KCH = KROW / 16;  // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* vbuf = smem;                                        // [STAGES][RS][VSTR]
  unsigned char* kbuf = vbuf + size_t(STAGES) * RS * VSTR;           // [STAGES][RS][KSTR]
  float* Dq = reinterpret_cast<float*>(kbuf + size_t(STAGES) * RS * KSTR);   // [16][WS]
  float* rp = Dq + kTileM * WS;                                      // [16][L+1]
  int* tgt = reinterpret_cast<int*>(rp + kTileM * (L + 1));          // [16]
  int* su = tgt + kTileM;                                            // [cap]
  uint32_t* smask = reinterpret_cast<uint32_t*>(su + p.plan.cap);    // [16][cap / 32 + 1]
  float* sw2 = reinterpret_cast<float*>(smask + kTileM * (p.plan.cap / 32 + 1));   // [P][C]
  uint64_t* fullbar = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(sw2 + (FUSED ? num_paths(L) * C : 0)) + 15) & ~uintptr_t(15));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(fullbar + STAGES);
  if (threadIdx.x == 0) {
    // one arrival per staged row of a stage; its bulk copies add the bytes
    for (int b = 0; b < STAGES; ++b) mbar_init(smem_u32(fullbar + b), RS);
    mbar_fence_init();
    *abort_flag = 0;
  }
  if constexpr (FUSED) {
    for (int e = threadIdx.x; e < num_paths(L) * C; e += H * 32) sw2[e] = __ldg(p.w2 + e);
  }

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int h = tid >> 5;           // this warp's head
  const int g = lane >> 2, t = lane & 3;
  const PlanView& pv = p.plan;
  const int words = pv.cap / 32;
  const int swords = words + 1;     // padded shared-memory mask row
  const char* hp_bytes = reinterpret_cast<const char*>(p.hp);
  const char* k_bytes = reinterpret_cast<const char*>(p.k);

  int gbase = 0;   // stages staged by this CTA before the current tile
  for (int tile = blockIdx.x; tile < pv.tiles; tile += gridDim.x) {
    const int U = pv.ulen[tile];
    const int nsteps = (U + kTileK - 1) / kTileK;         // k-steps of 16 union rows
    const int nstages = (nsteps + KS - 1) / KS;
    // the plan pads the union to whole k-steps; here it is padded further to
    // whole stages with its first atom, whose mask bits there are zero
    const int ustep = nsteps * kTileK;
    const int* __restrict__ uni = pv.uni + (long long)tile * pv.cap;
    const uint32_t* __restrict__ mrow = pv.mask + (long long)tile * words * kTileM;

    {
      constexpr int RW = kTileM * (1 + (L + 1) + WS);
      const float* R = pv.rec + (long long)tile * RW;
      if (tid < kTileM) tgt[tid] = reinterpret_cast<const int*>(R)[tid];
      if constexpr (FUSED) {
        for (int e = tid; e < kTileM * (L + 1); e += NTHR) rp[e] = R[kTileM + e];
        for (int e = tid; e < kTileM * WS; e += NTHR) Dq[e] = R[kTileM * (2 + L) + e];
      }
    }
    // the tile's union indices and membership mask into shared memory
    const int upad = nstages * RS;
    const int uw = (ustep + 31) / 32;   // mask words the plan wrote
    for (int e = tid; e < upad; e += NTHR) su[e] = uni[e < ustep ? e : 0];
    for (int e = tid; e < kTileM * uw; e += NTHR) {
      const int r = e / uw, w = e % uw;
      smask[r * swords + w] = mrow[w * kTileM + r];
    }
    if (upad > 32 * uw && tid < kTileM) smask[tid * swords + uw] = 0u;
    __syncthreads();   // tgt, su, smask visible

    // 32 threads per staged row; each copies chunks lane, lane + 32, ... of
    // the row's value and key bytes (rows past the padded union are skipped)
    // one thread per staged row: its value row and key row as two bulk copies
    // whose bytes complete the stage buffer's mbarrier phase
    auto issue = [&](int stage) {
      const int gs = gbase + stage;
      const int buf = gs % STAGES;
      constexpr int RSTRIDE = NTHR / RS;
      if (tid % RSTRIDE == 0) {
        const int r = tid / RSTRIDE;
        const long long atom = su[stage * RS + r];
        const uint32_t bar = smem_u32(fullbar + buf);
        mbar_arrive_expect_tx(bar, ROW + KROW);
        bulk_g2s(smem_u32(vbuf + (size_t(buf) * RS + r) * VSTR), hp_bytes + atom * ROW, ROW, bar);
        bulk_g2s(smem_u32(kbuf + (size_t(buf) * RS + r) * KSTR), k_bytes + atom * KROW, KROW, bar);
      }
    };
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s)
      if (s < nstages) issue(s);

    // Q fragment of this head for the tile's 16 targets
    uint32_t qa[4];
    {
      const int t0 = tgt[g], t1 = tgt[g + 8];
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
      qa[0] = t0 >= 0 ? __ldg(q32 + ((size_t)t0 * H * 16 + h * 16 + 2 * t) / 2) : 0u;
      qa[1] = t1 >= 0 ? __ldg(q32 + ((size_t)t1 * H * 16 + h * 16 + 2 * t) / 2) : 0u;
      qa[2] = t0 >= 0 ? __ldg(q32 + ((size_t)t0 * H * 16 + h * 16 + 2 * t + 8) / 2) : 0u;
      qa[3] = t1 >= 0 ? __ldg(q32 + ((size_t)t1 * H * 16 + h * 16 + 2 * t + 8) / 2) : 0u;
    }
    float acc[D][4];
#pragma unroll
    for (int d = 0; d < D; ++d)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[d][e] = 0.f;
    // zacc: P times an all-ones B fragment, i.e. the row sums of exactly the
    // bf16 weights the P V product uses (zacc[0] row g, zacc[2] row g+8)
    float zacc[4] = {0.f, 0.f, 0.f, 0.f};
    constexpr uint32_t kOnes = 0x3f803f80u;   // bf16x2 (1, 1)
    // reference maxima (log2 domain): a finite sentinel, so that a masked
    // entry (-inf) gives exp2(-inf) = 0 without a select
    constexpr float kNone = -1e30f;
    float mref0 = kNone, mref1 = kNone;
    constexpr float kLazy = 8.f;
    const float qs = p.qscale;
    const float inv_qs = 1.f / qs;
    // raw-logit thresholds that trigger a raise; start below any finite logit
    float thr0 = -INFINITY, thr1 = -INFINITY;

    for (int st = 0; st < nstages; ++st) {
      __syncthreads();   // every warp is done with the buffer about to be refilled
      if (st + STAGES - 1 < nstages) issue(st + STAGES - 1);
      const int buf = (gbase + st) % STAGES;
      bounded_wait(smem_u32(fullbar + buf), uint32_t((gbase + st) / STAGES) & 1u, kWaitPolls,
                   abort_flag);
      // ---- S = Q K^T for every k-step of the stage (stages are whole:
      // the union is padded to a multiple of RS rows)
      float sf[KS][2][4];
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        const uint32_t kb = smem_u32(kbuf + (size_t(buf) * RS + j * kTileK) * KSTR);
        uint32_t kf[4];
        const int row = (lane & 7) + 8 * (lane >> 4);
        const int half = (lane >> 3) & 1;
        ldsm_x4(kf, kb + row * KSTR + h * 32 + half * 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) sf[j][0][e] = sf[j][1][e] = 0.f;
        mma_bf16(sf[j][0], qa, kf[0], kf[1]);
        mma_bf16(sf[j][1], qa, kf[2], kf[3]);
      }
      // ---- mask (rows g and g+8 of the tile; bit k <-> union atom ub + k);
      // the stage's RS <= 32 bits sit in one mask word
      const int ub = st * RS;
      const uint32_t m0 = smask[g * swords + (ub >> 5)] >> ((ub & 31) + 2 * t);
      const uint32_t m1 = smask[(g + 8) * swords + (ub >> 5)] >> ((ub & 31) + 2 * t);
      float v[KS][8];   // raw logits; row g: cols 2t, 2t+1, 8+2t, 9+2t ; row g+8: same
      bool over = false;
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        const uint32_t w0 = m0 >> (16 * j), w1 = m1 >> (16 * j);
        v[j][0] = (w0 & 1u) ? sf[j][0][0] : -INFINITY;
        v[j][1] = (w0 & 2u) ? sf[j][0][1] : -INFINITY;
        v[j][2] = (w0 & 0x100u) ? sf[j][1][0] : -INFINITY;
        v[j][3] = (w0 & 0x200u) ? sf[j][1][1] : -INFINITY;
        v[j][4] = (w1 & 1u) ? sf[j][0][2] : -INFINITY;
        v[j][5] = (w1 & 2u) ? sf[j][0][3] : -INFINITY;
        v[j][6] = (w1 & 0x100u) ? sf[j][1][2] : -INFINITY;
        v[j][7] = (w1 & 0x200u) ? sf[j][1][3] : -INFINITY;
        over |= (v[j][0] > thr0) | (v[j][1] > thr0) | (v[j][2] > thr0) | (v[j][3] > thr0) |
                (v[j][4] > thr1) | (v[j][5] > thr1) | (v[j][6] > thr1) | (v[j][7] > thr1);
      }
      // ---- online softmax, one test per stage.  Common case: no logit of
      // the warp's rows exceeds its row's raw threshold (mref + kLazy) / qs,
      // tested per entry with no cross-lane traffic.  Otherwise the row
      // maxima over the stage are formed exactly and the rows that need it
      // are rescaled.
      if (__any_sync(0xffffffffu, over)) {
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
          mx0 = fmaxf(mx0, fmaxf(fmaxf(v[j][0], v[j][1]), fmaxf(v[j][2], v[j][3])));
          mx1 = fmaxf(mx1, fmaxf(fmaxf(v[j][4], v[j][5]), fmaxf(v[j][6], v[j][7])));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        mx0 *= qs;
        mx1 *= qs;
        const bool r0 = mx0 > mref0 + kLazy, r1 = mx1 > mref1 + kLazy;
        const float sc0 = r0 ? fast_exp2(mref0 - mx0) : 1.f;
        const float sc1 = r1 ? fast_exp2(mref1 - mx1) : 1.f;
        zacc[0] *= sc0;
        zacc[1] *= sc0;
        zacc[2] *= sc1;
        zacc[3] *= sc1;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          acc[d][0] *= sc0;
          acc[d][1] *= sc0;
          acc[d][2] *= sc1;
          acc[d][3] *= sc1;
        }
        if (r0) {
          mref0 = mx0;
          thr0 = (mref0 + kLazy) * inv_qs;
        }
        if (r1) {
          mref1 = mx1;
          thr1 = (mref1 + kLazy) * inv_qs;
        }
      }
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        float pr[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(fmaf(v[j][e], qs, -mref0));
#pragma unroll
        for (int e = 4; e < 8; ++e) pr[e] = fast_exp2(fmaf(v[j][e], qs, -mref1));
        uint32_t pa[4];
        {
          __nv_bfloat162 b;
          b = __floats2bfloat162_rn(pr[0], pr[1]); pa[0] = *reinterpret_cast<uint32_t*>(&b);  // row g,   k 2t
          b = __floats2bfloat162_rn(pr[4], pr[5]); pa[1] = *reinterpret_cast<uint32_t*>(&b);  // row g+8, k 2t
          b = __floats2bfloat162_rn(pr[2], pr[3]); pa[2] = *reinterpret_cast<uint32_t*>(&b);  // row g,   k 2t+8
          b = __floats2bfloat162_rn(pr[6], pr[7]); pa[3] = *reinterpret_cast<uint32_t*>(&b);  // row g+8, k 2t+8
        }
        mma_bf16(zacc, pa, kOnes, kOnes);

        // ---- O += P V (one n8 tile per component of this head's 8 channels)
        const uint32_t vb = smem_u32(vbuf + (size_t(buf) * RS + j * kTileK) * VSTR);
        const int mj = lane >> 3;                 // matrix of this lane's row address
        const int row = (lane & 7) + 8 * (mj & 1);
        const uint32_t base = vb + row * VSTR + h * 16;
#pragma unroll
        for (int d = 0; d + 1 < D; d += 2) {
          uint32_t vf[4];
          ldsm_x4_t(vf, base + (d + (mj >> 1)) * (C * 2));
          mma_bf16(acc[d], pa, vf[0], vf[1]);
          mma_bf16(acc[d + 1], pa, vf[2], vf[3]);
        }
        if constexpr (D % 2) {
          uint32_t vf[2];
          ldsm_x2_t(vf, base + (D - 1) * (C * 2));
          mma_bf16(acc[D - 1], pa, vf[0], vf[1]);
        }
      }   // k-steps of the stage
    }
    __syncthreads();   // all staged buffers consumed
    gbase += nstages;

    // ---- epilogue: normalise; either write m or apply the target coupling
    const float inv0 = zacc[0] > 0.f ? 1.f / zacc[0] : 0.f;
    const float inv1 = zacc[2] > 0.f ? 1.f / zacc[2] : 0.f;
    const int ch = h * 8 + 2 * t;
    if constexpr (FUSED && L >= 3) {
      // register budget: m of both rows goes through this warp's slice of the
      // drained staging buffers (8 KB per warp) so the accumulators are free
      // before the coupling; one channel at a time, scalar stores
      float* mw = reinterpret_cast<float*>(vbuf) + h * (kTileM * D * 8);
#pragma unroll
      for (int d = 0; d < D; ++d) {
        *reinterpret_cast<float2*>(mw + (g * D + d) * 8 + 2 * t) =
            make_float2(acc[d][0] * inv0, acc[d][1] * inv0);
        *reinterpret_cast<float2*>(mw + ((g + 8) * D + d) * 8 + 2 * t) =
            make_float2(acc[d][2] * inv1, acc[d][3] * inv1);
      }
      __syncwarp();
#pragma unroll 1
      for (int pr = 0; pr < 4; ++pr) {
        const int r = g + 8 * (pr >> 1), e = pr & 1;
        const int tg = tgt[r];
        if (tg < 0) continue;
        float rpow[L + 1];
#pragma unroll
        for (int l = 0; l <= L; ++l) rpow[l] = rp[r * (L + 1) + l];
        float x[D];
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] = mw[(r * D + d) * 8 + 2 * t + e];
        float* o = p.out + (size_t)tg * D * C + ch + e;
        eaas_channel<L>(x, Dq + r * WS, rpow, p.tab,
                        [&](int pp) { return sw2[pp * C + ch + e]; },
                        [&](int d, float val) { o[d * C] = val; });
      }
    } else
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = g + 8 * half;
      const int tg = tgt[r];
      if (tg < 0) continue;
      const float inv = half ? inv1 : inv0;
      float* o = p.out + (size_t)tg * D * C + ch;
      if constexpr (!FUSED) {
#pragma unroll
        for (int d = 0; d < D; ++d)
          *reinterpret_cast<float2*>(o + d * C) =
              make_float2(acc[d][2 * half] * inv, acc[d][2 * half + 1] * inv);
      } else {
        float rpow[L + 1];
#pragma unroll
        for (int l = 0; l <= L; ++l) rpow[l] = rp[r * (L + 1) + l];
        // channels 2t and 2t+1 of one target share its Wigner-D matrices
        float x[2][D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
          x[0][d] = acc[d][2 * half] * inv;
          x[1][d] = acc[d][2 * half + 1] * inv;
        }
        eaas_multi<L, 2>(x, Dq + r * WS, rpow, p.tab,
                         [&](int pp, int k) { return sw2[pp * C + ch + k]; },
                         [&](int d, const float (&y)[2]) {
                           *reinterpret_cast<float2*>(o + d * C) = make_float2(y[0], y[1]);
                         });
      }
    }
    if constexpr (FUSED && L >= 3) fence_proxy_async_smem();   // scratch before bulk copies
    __syncthreads();   // tgt / Dq / rp are rewritten by the next tile
  }
  if (*abort_flag && threadIdx.x == 0) {
    // a wait gave up: give each buffer's last fill a short, bounded chance to
    // land before the CTA's shared memory is released
    volatile int none = 0;
    for (int b = 0; b < STAGES && b < gbase; ++b)
      bounded_wait(smem_u32(fullbar + b), uint32_t((gbase - 1 - b) / STAGES) & 1u, kDrainPolls, &none);
  }
}

// A wait that cannot succeed: one arrival announces 16 bytes that no copy
// will deliver, so the phase never completes and bounded_wait must give up
// after `polls` polls — exercises the timeout report without any fault.
__global__ void wait_timeout_selftest_kernel(int polls) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(smem_u32(&bar), 16);
    bounded_wait(smem_u32(&bar), 0u, polls, &abort_flag);
  }
}

template <int L, int H, bool FUSED>
int launch_tc_t(const TcParams& p, int tiles, cudaStream_t st) {
  const size_t shmem = tc_smem_fixed<L, H>() + tc_smem_plan(p.plan.cap) +
                       (FUSED ? tc_smem_w2<L, H>() : 0) + kBarBytes;
  if (shmem > 227 * 1024) return EGAT_ERR_UNSUPPORTED;
  auto kern = otf_attention_tc_kernel<L, H, FUSED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shmem)) !=
      cudaSuccess)
    return EGAT_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = tiles < sms ? tiles : sms;
  kern<<<grid, H * 32, shmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace

bool tc_attention_supported(const egat_shape& s) {
  if (!(s.dtype == EGAT_BF16 && s.graph_mode == EGAT_GRAPH_PADDED && s.dk == 16 && s.H == 16 &&
        s.C == 128 && s.lmax >= 1 && s.lmax <= 3))
    return false;
  if (plan_smem_bytes(s.n, s.K) > kPlanSmemLimit) return false;
  const size_t fixed = s.lmax == 1 ? tc_smem_fixed<1, 16>()
                     : s.lmax == 2 ? tc_smem_fixed<2, 16>() : tc_smem_fixed<3, 16>();
  const size_t w2 = s.lmax == 1 ? tc_smem_w2<1, 16>()
                  : s.lmax == 2 ? tc_smem_w2<2, 16>() : tc_smem_w2<3, 16>();
  return fixed + tc_smem_plan(plan_capacity(s.K)) + w2 + kBarBytes <= 227 * 1024;
}

int launch_attention_tc(const egat_shape& s, bool fused, const void* d_q, const void* d_k,
                        const void* d_hp, const void* d_plan, const float* d_w2, float* d_out,
                        cudaStream_t st) {
  if (!tc_attention_supported(s)) return EGAT_ERR_UNSUPPORTED;
  TcParams p;
  p.q = static_cast<const __nv_bfloat16*>(d_q);
  p.k = static_cast<const __nv_bfloat16*>(d_k);
  p.hp = static_cast<const __nv_bfloat16*>(d_hp);
  p.plan = plan_view(const_cast<void*>(d_plan), s.n, s.K, s.lmax);
  p.order = nullptr;
  p.out = d_out;
  p.pos = nullptr;
  p.w2 = d_w2;
  p.n = s.n;
  p.qscale = float(1.4426950408889634 / std::sqrt(double(s.dk)));
  if (fused) p.tab = eaas_table(s.lmax);
  else memset(&p.tab, 0, sizeof(p.tab));
  const int tiles = p.plan.tiles;
  switch (s.lmax) {
    case 1: return fused ? launch_tc_t<1, 16, true>(p, tiles, st) : launch_tc_t<1, 16, false>(p, tiles, st);
    case 2: return fused ? launch_tc_t<2, 16, true>(p, tiles, st) : launch_tc_t<2, 16, false>(p, tiles, st);
    case 3: return fused ? launch_tc_t<3, 16, true>(p, tiles, st) : launch_tc_t<3, 16, false>(p, tiles, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

int take_wait_timeouts(cudaStream_t st, unsigned int* count) {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_wait_timeouts) != cudaSuccess) return EGAT_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyAsync(&h, addr, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(addr, 0, sizeof(h), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return EGAT_ERR_CUDA;
  *count = h;
  return EGAT_OK;
}

int launch_wait_timeout_selftest(int polls, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(polls);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
