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
//    one reference;
//  * the float32 weights p become two bf16 A fragments, hi = bf16(p) and
//    lo = bf16(p - hi) (the S fragment layout of two n8 tiles is the A layout
//    of one k16 step), so P V carries p to about 2^-17 rather than bf16's
//    2^-9: P V_h runs as two mma.sync per component of the head's 8 channels
//    (the lo products one component pair behind the hi ones, off the same
//    accumulator's dependency chain), the value fragments by ldmatrix.trans
//    from the staged rows; z is the float32 row sum of the weights, on the
//    FMA pipe (the pairs equal the weights to about 2^-17), which keeps the
//    busier tensor pipe for the products.
// The accumulator fragment of a lane holds, for targets g and g+8 and
// channels 2t, 2t+1 of its head, every component d — exactly what the
// per-channel EAAS epilogue needs, so the target coupling runs from registers.
#include <cfloat>

#include "egat_async.cuh"
#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kRowPad = 16;   // bytes of padding per staged row

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

// max(a, b, c) in one instruction (the three-input form of sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (a, b) as bf16x2 pairs hi + lo with hi = bf16(x) and lo = bf16(x - hi),
// both rounded to nearest even: hi + lo equals x to about 2^-17 relative
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  hi = *reinterpret_cast<uint32_t*>(&h);
  // (a, b) - float(hi) as one packed f32x2 FMA
  const f32x2 r = f2_fma(bf16x2_to_f2(hi), f2_pack(-1.f, -1.f), f2_pack(a, b));
  float ra, rb;
  f2_unpack(r, ra, rb);
  __nv_bfloat162 l = __floats2bfloat162_rn(ra, rb);
  lo = *reinterpret_cast<uint32_t*>(&l);
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

// Shared-memory layout (byte offsets; every region 16-byte aligned): staged
// value and key rows, the tile's query rows, two tile records (current and
// next), the target-coupling weights [P][C] (fused), the mbarriers, the
// abort flag and the claimed next tile, then the tile's union indices [cap] and word-major membership
// mask [cap / 32][16] (6 cap bytes, sized at launch).
template <int L, int H, bool FUSED>
struct TcSmem {
  using Sh = TcShape<L>;
  static constexpr int D = Sh::D, C = 8 * H;
  static constexpr int VSTR = D * C * 2 + kRowPad;   // staged value row
  static constexpr int KSTR = H * 32 + kRowPad;      // staged key row (dk = 16)
  static constexpr int QSTR = KSTR;                  // staged query row
  static constexpr int REC = plan_record_words(L);
  static_assert(REC % 4 == 0, "records move in 16-byte units");
  static constexpr int NBARS = Sh::STAGES + 4;       // rows [STAGES], record [2], indices, mask
  static constexpr size_t vbuf = 0;
  static constexpr size_t kbuf = vbuf + size_t(Sh::STAGES) * Sh::RS * VSTR;
  static constexpr size_t sq = kbuf + size_t(Sh::STAGES) * Sh::RS * KSTR;
  static constexpr size_t rec = sq + size_t(kTileM) * QSTR;
  static constexpr size_t sw2 = rec + 2 * size_t(REC) * 4;
  static constexpr size_t bars = sw2 + (FUSED ? size_t(num_paths(L)) * C * 4 : 0);
  static constexpr size_t su = bars + (size_t(NBARS) * 8 + 8 + 15) / 16 * 16;   // + abort flag, next tile
  static size_t total(int cap) { return su + size_t(cap) * 4 + size_t(cap / 32) * kTileM * 4; }
};
// the fused epilogue at lmax >= 3 keeps m of the tile in the stage buffers
template <int L, int H>
constexpr bool tc_scratch_fits() {
  return size_t(H) * kTileM * TcShape<L>::D * 8 * 4 <=
         size_t(TcShape<L>::STAGES) * TcShape<L>::RS * TcSmem<L, H, true>::VSTR;
}
static_assert(tc_scratch_fits<3, 16>(), "lmax 3 epilogue scratch");

template <int L, int H, bool FUSED>
__global__ void __launch_bounds__(H * 32, 1)
otf_attention_tc_kernel(const __grid_constant__ TcParams p) {
  using Sm = TcSmem<L, H, FUSED>;
  constexpr int D = (L + 1) * (L + 1);
  constexpr int C = 8 * H;
  constexpr int ROW = D * C * 2;                  // value row bytes
  constexpr int VSTR = Sm::VSTR;
  constexpr int KROW = H * 16 * 2;                // key / query row bytes (dk = 16)
  constexpr int KSTR = Sm::KSTR;
  constexpr int QSTR = Sm::QSTR;
  constexpr int STAGES = TcShape<L>::STAGES;
  constexpr int KS = TcShape<L>::KS;
  constexpr int RS = TcShape<L>::RS;
  constexpr int REC = Sm::REC;
  constexpr int WS = wig_size(L);
  constexpr int NTHR = H * 32;
  // the fused lmax 3 epilogue uses the stage buffers as scratch, so there the
  // next tile's first rows are staged after it
  constexpr bool kEarlyRows = !(FUSED && L >= 3);
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* vbuf = smem + Sm::vbuf;                                 // [STAGES][RS][VSTR]
  unsigned char* kbuf = smem + Sm::kbuf;                                 // [STAGES][RS][KSTR]
  unsigned char* sq = smem + Sm::sq;                                     // [16][QSTR]
  float* recbuf = reinterpret_cast<float*>(smem + Sm::rec);              // [2][REC]
  float* sw2 = reinterpret_cast<float*>(smem + Sm::sw2);                 // [P][C]
  uint64_t* fullbar = reinterpret_cast<uint64_t*>(smem + Sm::bars);      // [STAGES] a stage's rows
  uint64_t* recbar = fullbar + STAGES;                                   // [2] a tile record
  uint64_t* idxbar = recbar + 2;                                         // a tile's indices + queries
  uint64_t* mskbar = idxbar + 1;                                         // a tile's mask
  volatile int* abort_flag = reinterpret_cast<volatile int*>(mskbar + 1);
  int* s_next = reinterpret_cast<int*>(mskbar + 1) + 1;                  // the CTA's next tile
  int* su = reinterpret_cast<int*>(smem + Sm::su);                       // [cap]
  uint32_t* smask = reinterpret_cast<uint32_t*>(su + p.plan.cap);        // [cap / 32][16]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int h = tid >> 5;           // this warp's head
  const int g = lane >> 2, t = lane & 3;
  const PlanView& pv = p.plan;
  const int words = pv.cap / 32;
  const int grid = gridDim.x;
  const char* hp_bytes = reinterpret_cast<const char*>(p.hp);
  const char* k_bytes = reinterpret_cast<const char*>(p.k);
  const char* q_bytes = reinterpret_cast<const char*>(p.q);
  // Tiles are claimed at run time (union sizes, hence tile costs, vary by
  // about a quarter): a CTA's first tile is blockIdx.x; near the end of each
  // tile thread 0 takes a ticket c from the plan's counter and the CTA's
  // next tile is grid + c (past the last tile: done).  Every processed tile
  // takes exactly one ticket, so a launch hands out tickets 0 .. tiles - 1,
  // in that order; the CTA holding the last one sets the counter back to
  // zero for the next launch on the plan (ordered after this one).
  if (blockIdx.x >= pv.tiles) return;   // whole CTA

  if (tid == 0) {
    // a stage buffer: one arrival per staged row, whose bulk copies add the
    // bytes; records, indices and masks: one arrival by the issuing thread
    for (int b = 0; b < STAGES; ++b) mbar_init(smem_u32(fullbar + b), RS);
    for (int b = 0; b < 4; ++b) mbar_init(smem_u32(recbar + b), 1);
    mbar_fence_init();
    *abort_flag = 0;
  }
  if constexpr (FUSED) {
    for (int e = tid; e < num_paths(L) * C; e += NTHR) sw2[e] = __ldg(p.w2 + e);
  }
  __syncthreads();

  // union length of a tile record, clamped so that a record that never
  // arrived (after a wait gave up) still gives bounded, in-range copies
  auto rec_ulen = [&](const float* rec) {
    const int U = reinterpret_cast<const int*>(rec)[0];
    return U < 0 ? 0 : (U > pv.cap ? pv.cap : U);
  };
  auto stages_of = [&](const float* rec) { return (rec_ulen(rec) + RS - 1) / RS; };
  // thread 0: a tile's record into recbuf[b]
  auto issue_record = [&](int tl, int b) {
    const uint32_t bar = smem_u32(recbar + b);
    mbar_arrive_expect_tx(bar, REC * 4);
    bulk_g2s(smem_u32(recbuf + b * REC), pv.rec + (long long)tl * REC, REC * 4, bar);
  };
  // thread 0: a tile's union indices (as the plan padded them) and the query
  // rows of its targets (atom 0's row for an empty slot; unused)
  auto issue_index = [&](int tl, const float* rec) {
    const int U = rec_ulen(rec);
    const int upad = U > 0 ? (U + kPlanPad - 1) / kPlanPad * kPlanPad : kPlanPad;
    const uint32_t bar = smem_u32(idxbar);
    mbar_arrive_expect_tx(bar, upad * 4 + kTileM * KROW);
    bulk_g2s(smem_u32(su), pv.uni + (long long)tl * pv.cap, upad * 4, bar);
    const int* tg = reinterpret_cast<const int*>(rec) + kRecTgt;
    for (int r = 0; r < kTileM; ++r) {
      const long long a = (unsigned)tg[r] < (unsigned)p.n ? tg[r] : 0;
      bulk_g2s(smem_u32(sq + r * QSTR), q_bytes + a * KROW, KROW, bar);
    }
  };
  // thread 0: a tile's membership mask (the words the plan wrote)
  auto issue_mask = [&](int tl, const float* rec) {
    const int U = rec_ulen(rec);
    const int uw = U > 0 ? (U + 31) / 32 : 1;
    const uint32_t bar = smem_u32(mskbar);
    mbar_arrive_expect_tx(bar, uw * kTileM * 4);
    bulk_g2s(smem_u32(smask), pv.mask + (long long)tl * words * kTileM, uw * kTileM * 4, bar);
  };
  // one thread per staged row: rows of tile-local stage s (global stage gs) as
  // two bulk copies whose bytes complete the stage buffer's mbarrier phase
  auto issue_rows = [&](int s, int gs) {
    const int buf = gs % STAGES;
    constexpr int RSTRIDE = NTHR / RS;
    if (tid % RSTRIDE == 0) {
      const int r = tid / RSTRIDE;
      long long atom = su[s * RS + r];
      if ((unsigned long long)atom >= (unsigned long long)p.n) atom = 0;
      const uint32_t bar = smem_u32(fullbar + buf);
      mbar_arrive_expect_tx(bar, ROW + KROW);
      bulk_g2s(smem_u32(vbuf + (size_t(buf) * RS + r) * VSTR), hp_bytes + atom * ROW, ROW, bar);
      bulk_g2s(smem_u32(kbuf + (size_t(buf) * RS + r) * KSTR), k_bytes + atom * KROW, KROW, bar);
    }
  };

  // first tile: record, then its indices, queries and mask, then its first rows
  int tile = blockIdx.x;
  int gbase = 0;   // stages staged by this CTA before the current tile
  if (tid == 0) issue_record(tile, 0);
  bounded_wait(smem_u32(recbar), 0u, kWaitPolls, abort_flag);
  if (tid == 0) {
    issue_index(tile, recbuf);
    issue_mask(tile, recbuf);
  }
  bounded_wait(smem_u32(idxbar), 0u, kWaitPolls, abort_flag);
  {
    const int ns = stages_of(recbuf);
    for (int s = 0; s < STAGES - 1 && s < ns; ++s) issue_rows(s, s);
  }

  int k = 0;   // this CTA's tile sequence number
  while (tile < pv.tiles) {
    const float* rec = recbuf + (k & 1) * REC;
    const float* nrec = recbuf + ((k + 1) & 1) * REC;
    // thread 0 claims the tile after this one a stage before it takes the
    // claim (the next tile's record copy), which is a stage before the next
    // tile's indices are copied; every thread learns the next tile after
    // the stage loop
    int ticket = 0;
    auto claim = [&]() { ticket = atomicAdd(pv.sched, 1); };
    int next = pv.tiles;
    bool has_next = false;
    // this tile's record, indices, queries and mask (all issued during the
    // previous tile, or above)
    bounded_wait(smem_u32(recbar + (k & 1)), uint32_t(k >> 1) & 1u, kWaitPolls, abort_flag);
    bounded_wait(smem_u32(idxbar), uint32_t(k) & 1u, kWaitPolls, abort_flag);
    bounded_wait(smem_u32(mskbar), uint32_t(k) & 1u, kWaitPolls, abort_flag);
    const int nstages = stages_of(rec);
    // thread 0: publish the claimed tile and copy its record into the other
    // buffer (its last reader, the previous tile's epilogue, finished before
    // that tile's last barrier)
    auto take_claim = [&]() {
      if (ticket == pv.tiles - 1) atomicExch(pv.sched, 0);   // every ticket was handed out
      next = grid + ticket;
      has_next = next < pv.tiles;
      *s_next = next;
      if (has_next) issue_record(next, (k + 1) & 1);
    };

    // Q fragment of this head for the tile's 16 targets
    uint32_t qa[4];
    {
      const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
      ldsm_x4(qa, smem_u32(sq + row * QSTR + h * 32 + (lane >> 4) * 16));
    }
    float acc[D][4];
#pragma unroll
    for (int d = 0; d < D; ++d)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[d][e] = 0.f;
    // z0, z1: this lane's float32 sums of the weights of rows g and g+8 (its
    // columns of the stage); the quad's four lanes are added at the tile's end.
    // The hi + lo pairs of P V equal these weights to about 2^-17.
    float z0 = 0.f, z1 = 0.f;
    // reference maxima (log2 domain): a finite sentinel, so that a masked
    // entry (-inf) gives exp2(-inf) = 0 without a select
    constexpr float kNone = -1e30f;
    float mref0 = kNone, mref1 = kNone;
    constexpr float kLazy = 8.f;
    const float qs = p.qscale;
    const float inv_qs = 1.f / qs;
    // raw-logit thresholds that trigger a raise; start below any finite logit
    float thr0 = -INFINITY, thr1 = -INFINITY;

    // the stage after which the indices and query rows are free for the next
    // tile: its barrier follows the last issue that reads them
    const int trig = nstages - STAGES + 1 > 0 ? nstages - STAGES + 1 : 0;
    const int take_st = trig > 1 ? trig - 1 : 0;     // the claim is taken no later than trig
    const int claim_st = take_st > 1 ? take_st - 1 : 0;
    for (int st = 0; st < nstages; ++st) {
      __syncthreads();   // every warp is done with the buffer about to be refilled
      if (st + STAGES - 1 < nstages) issue_rows(st + STAGES - 1, gbase + st + STAGES - 1);
      if (st == claim_st && tid == 0) claim();
      if (st == take_st && tid == 0) take_claim();
      if (st == trig && tid == 0 && has_next) {
        bounded_wait(smem_u32(recbar + ((k + 1) & 1)), uint32_t((k + 1) >> 1) & 1u, kWaitPolls,
                     abort_flag);
        issue_index(next, nrec);
      }
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
      const uint32_t m0 = smask[(ub >> 5) * kTileM + g] >> ((ub & 31) + 2 * t);
      const uint32_t m1 = smask[(ub >> 5) * kTileM + g + 8] >> ((ub & 31) + 2 * t);
      float v[KS][8];   // raw logits; row g: cols 2t, 2t+1, 8+2t, 9+2t ; row g+8: same
      float lm0 = -INFINITY, lm1 = -INFINITY;   // this lane's largest logit of rows g, g+8
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
        lm0 = max3f(max3f(lm0, v[j][0], v[j][1]), v[j][2], v[j][3]);
        lm1 = max3f(max3f(lm1, v[j][4], v[j][5]), v[j][6], v[j][7]);
      }
      const bool over = (lm0 > thr0) | (lm1 > thr1);
      // ---- online softmax, one test per stage.  Common case: no logit of
      // the warp's rows exceeds its row's raw threshold (mref + kLazy) / qs,
      // tested on the lane's row maxima with no cross-lane traffic.
      // Otherwise the row maxima over the stage are completed across the
      // quad and the rows that need it are rescaled.
      if (__any_sync(0xffffffffu, over)) {
        float mx0 = lm0, mx1 = lm1;
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        mx0 *= qs;
        mx1 *= qs;
        const bool r0 = mx0 > mref0 + kLazy, r1 = mx1 > mref1 + kLazy;
        const float sc0 = r0 ? fast_exp2(mref0 - mx0) : 1.f;
        const float sc1 = r1 ? fast_exp2(mref1 - mx1) : 1.f;
        z0 *= sc0;
        z1 *= sc1;
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
        {
          // exponents v qs - mref as packed f32x2 FMAs (pairs of one row)
          const f32x2 q2 = f2_pack(qs, qs);
          const f32x2 r0 = f2_pack(-mref0, -mref0), r1 = f2_pack(-mref1, -mref1);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const f32x2 x = f2_fma(f2_pack(v[j][e], v[j][e + 1]), q2, e < 4 ? r0 : r1);
            float x0, x1;
            f2_unpack(x, x0, x1);
            pr[e] = fast_exp2(x0);
            pr[e + 1] = fast_exp2(x1);
          }
        }
        // the weights as a bf16 pair hi + lo (hi = bf16(p), lo = bf16(p - hi)):
        // 16 significant bits, so P V and the normaliser carry the float32
        // weights to about 2^-17 instead of bf16's 2^-9
        uint32_t pa[4], pl[4];
        split_bf16(pr[0], pr[1], pa[0], pl[0]);   // row g,   k 2t
        split_bf16(pr[4], pr[5], pa[1], pl[1]);   // row g+8, k 2t
        split_bf16(pr[2], pr[3], pa[2], pl[2]);   // row g,   k 2t+8
        split_bf16(pr[6], pr[7], pa[3], pl[3]);   // row g+8, k 2t+8
        z0 += (pr[0] + pr[1]) + (pr[2] + pr[3]);
        z1 += (pr[4] + pr[5]) + (pr[6] + pr[7]);

        // ---- O += P V (one n8 tile per component of this head's 8 channels).
        // The lo products run one component pair behind the hi products, so
        // that no mma waits on the one just issued into the same accumulator.
        const uint32_t vb = smem_u32(vbuf + (size_t(buf) * RS + j * kTileK) * VSTR);
        const int mj = lane >> 3;                 // matrix of this lane's row address
        const int row = (lane & 7) + 8 * (mj & 1);
        const uint32_t base = vb + row * VSTR + h * 16;
        uint32_t vprev[4];
#pragma unroll
        for (int d = 0; d + 1 < D; d += 2) {
          uint32_t vf[4];
          ldsm_x4_t(vf, base + (d + (mj >> 1)) * (C * 2));
          mma_bf16(acc[d], pa, vf[0], vf[1]);
          mma_bf16(acc[d + 1], pa, vf[2], vf[3]);
          if (d >= 2) {
            mma_bf16(acc[d - 2], pl, vprev[0], vprev[1]);
            mma_bf16(acc[d - 1], pl, vprev[2], vprev[3]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) vprev[e] = vf[e];
        }
        if constexpr (D % 2) {
          uint32_t vf[2];
          ldsm_x2_t(vf, base + (D - 1) * (C * 2));
          mma_bf16(acc[D - 1], pa, vf[0], vf[1]);
          if constexpr (D > 1) {
            mma_bf16(acc[D - 3], pl, vprev[0], vprev[1]);
            mma_bf16(acc[D - 2], pl, vprev[2], vprev[3]);
          }
          mma_bf16(acc[D - 1], pl, vf[0], vf[1]);
        } else {
          mma_bf16(acc[D - 2], pl, vprev[0], vprev[1]);
          mma_bf16(acc[D - 1], pl, vprev[2], vprev[3]);
        }
      }   // k-steps of the stage
    }
    if (nstages == 0 && tid == 0) {
      claim();
      take_claim();
    }
    __syncthreads();   // every warp is done with the stage buffers and the mask
    next = *s_next;    // rewritten only after the tile's last barrier
    has_next = next < pv.tiles;
    gbase += nstages;
    if (tid == 0 && has_next) {
      if (nstages == 0) {
        bounded_wait(smem_u32(recbar + ((k + 1) & 1)), uint32_t((k + 1) >> 1) & 1u, kWaitPolls,
                     abort_flag);
        issue_index(next, nrec);
      }
      issue_mask(next, nrec);
    }
    // the next tile's first rows (needs its record and indices)
    auto stage_next = [&]() {
      bounded_wait(smem_u32(recbar + ((k + 1) & 1)), uint32_t((k + 1) >> 1) & 1u, kWaitPolls,
                   abort_flag);
      bounded_wait(smem_u32(idxbar), uint32_t(k + 1) & 1u, kWaitPolls, abort_flag);
      const int ns = stages_of(nrec);
      for (int s = 0; s < STAGES - 1 && s < ns; ++s) issue_rows(s, gbase + s);
    };
    if (kEarlyRows && has_next) stage_next();

    // ---- epilogue of the tile: normalise; either write m or apply the target
    // coupling (the next tile's first rows are already in flight, except at
    // fused lmax 3)
    const int* tgt = reinterpret_cast<const int*>(rec) + kRecTgt;
    const float* rp = rec + kRecRp;             // [16][L+1]
    const float* Dq = rec + rec_off_D(L);       // [16][WS]
    z0 += __shfl_xor_sync(0xffffffffu, z0, 1);
    z0 += __shfl_xor_sync(0xffffffffu, z0, 2);
    z1 += __shfl_xor_sync(0xffffffffu, z1, 1);
    z1 += __shfl_xor_sync(0xffffffffu, z1, 2);
    const float inv0 = z0 > 0.f ? 1.f / z0 : 0.f;
    const float inv1 = z1 > 0.f ? 1.f / z1 : 0.f;
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
    if constexpr (!kEarlyRows) fence_proxy_async_smem();   // scratch before bulk copies
    __syncthreads();   // the record buffer and the stage buffers are refilled next
    if (!kEarlyRows && has_next) stage_next();
    ++k;
    tile = next;
  }
  if (*abort_flag && tid == 0) {
    // a wait gave up: give every barrier's last phase a short, bounded chance
    // to complete before the CTA's shared memory is released
    volatile int none = 0;
    for (int b = 0; b < STAGES && b < gbase; ++b)
      bounded_wait(smem_u32(fullbar + b), uint32_t((gbase - 1 - b) / STAGES) & 1u, kDrainPolls,
                   &none);
    for (int b = 0; b < 2; ++b) {
      const int last = k - 1 - ((k - 1 - b) & 1);   // last tile sequence number of parity b
      if (last >= 0) bounded_wait(smem_u32(recbar + b), uint32_t(last >> 1) & 1u, kDrainPolls, &none);
    }
    if (k > 0) {
      bounded_wait(smem_u32(idxbar), uint32_t(k - 1) & 1u, kDrainPolls, &none);
      bounded_wait(smem_u32(mskbar), uint32_t(k - 1) & 1u, kDrainPolls, &none);
    }
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
  const size_t shmem = TcSmem<L, H, FUSED>::total(p.plan.cap);
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
  const int cap = plan_capacity(s.K);
  const size_t smem = s.lmax == 1 ? TcSmem<1, 16, true>::total(cap)
                    : s.lmax == 2 ? TcSmem<2, 16, true>::total(cap) : TcSmem<3, 16, true>::total(cap);
  return smem <= 227 * 1024;
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

int take_wait_timeouts_attention(cudaStream_t st, unsigned int* count) {
  return take_unit_wait_timeouts(st, count) == 0 ? EGAT_OK : EGAT_ERR_CUDA;
}

int launch_wait_timeout_selftest(int polls, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(polls);
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
