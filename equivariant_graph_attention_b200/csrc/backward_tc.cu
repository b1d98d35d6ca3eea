// Tiled tensor-core passes of the backward pass (bf16 storage, C = 128,
// H = 16, dk = 16): the attention gradients dq, dk and dh' of
// L = sum_i <G_i, ^h_i>, every attention weight recomputed, nothing per edge
// stored ("E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.2, linear
// activation memory; "E2Former-V2: On-the-Fly Equivariant Attention with
// Linear Activation Memory" §2.2).
//
// With lse_i the log-sum-exp of target i's logits (per head), alpha_ij =
// 2^(s_ij qs - lse_i) exactly, and per head
//   dalpha_ij = <dm_i, h'_j>                 (the head's 8 channels x D components)
//   Delta_i   = sum_j alpha_ij dalpha_ij
//   ds_ij     = alpha_ij (dalpha_ij - Delta_i)
//   dq_i      = sum_j ds_ij k_j / sqrt(dk)   = (A_i - Delta_i B_i) / sqrt(dk),
//               A_i = sum_j alpha dalpha k_j,  B_i = sum_j alpha k_j
//   dk_j      = sum_i ds_ij q_i / sqrt(dk),  dh'_j = sum_i alpha_ij dm_i.
//
// Three passes, each over tiles of 16 atoms that share one streamed union:
//  * statistics pass: the forward's tiles (16 targets, the union of their
//    neighbour lists, membership mask) and the forward's online softmax, but
//    P H' in tf32 and the weight sums in float32: m_i (which dL/dr needs) and
//    lse_i.  The forward's own bf16 operands would give m to 4e-3 and
//    normalise alpha to 2e-3 only, and dq = A - Delta B cancels that error
//    up by an order of magnitude;
//  * target pass: the same tiles; per 8 union atoms and head, S = Q K^T
//    (bf16 mma), dalpha = dm H'^T, A += (alpha dalpha) K and B += alpha K
//    (tf32 mma); dq and Delta in the epilogue, one sweep;
//  * source pass: tiles of 16 sources and the union of the targets whose
//    lists hold them (in-lists, bitmap union as for the forward plan); per 8
//    union targets and head, S^T = K Q^T, dalpha^T = H' dm^T,
//    dk += ds^T Q and dh' += alpha^T dm.
// At lmax 3 (16 components: 8 KB float rows) a stage holds 8 union rows, and
// the source pass sweeps its union twice, once for dk (with h' as the
// register-resident operand) and once for dh' (with its accumulator), since
// the two would not fit one thread's registers together.
// The tile's own operand (dm of the 16 targets, or h' of the 16 sources) sits
// in registers as tf32 fragments for the whole tile; the union rows stream
// through shared memory in stages, one bulk copy (cp.async.bulk, no
// multicast) per row and array completing the stage's mbarrier, every wait
// bounded.  The softmax derivative subtracts nearly equal numbers, so its
// operands are float32 rounded to tf32 (10-bit mantissa), not bf16: the
// modelled error of dq on the 4,096-atom workload is 3e-3 of the row norm.
// dh' = alpha^T dm feeds the adjoint source coupling, whose |r|^l-scaled
// terms cancel on small channels of dL/dh; there both operands enter as tf32
// pairs hi + lo (three products), so dh' carries float32-level accuracy.
// Every sum runs in a fixed order (union order, then the stage's k-steps):
// deterministic, no atomics on results.
#include <cfloat>
#include <cmath>

#include "egat_async.cuh"
#include "egat_device.cuh"
#include "egat_host.h"

namespace egat {
namespace {

constexpr int kBH = 16;                 // heads (one warp each)
constexpr int kBC = 128;                // channels
constexpr int kBThreads = kBH * 32;
constexpr int kKRow = kBH * 16 * 2;     // q / k row bytes (dk = 16, bf16)
constexpr int kKStr = kKRow + 16;       // staged q / k row (padded: distinct ldmatrix banks)
constexpr int kSRow = 2 * kBH * 4;      // stats row: lse[H], Delta[H] (float)
constexpr int kSStr = kSRow + 16;

template <int L>
struct BtcShape {
  static constexpr int D = (L + 1) * (L + 1);
  static constexpr int FROW = D * kBC * 4;      // float32 row of h' or dm
  static constexpr int FSTR = FROW + 16;        // staged (4 words mod 32: distinct banks)
  // union rows per stage: two n8 tiles, one at lmax 3 (8 KB float rows)
  static constexpr int RS = L >= 3 ? 8 : 16;
  static constexpr int STAGES = L >= 3 ? 3 : (L >= 2 ? 2 : 4);
};

// Shared memory (byte offsets, 16-byte aligned): staged float rows (FR),
// staged q / k rows, staged stats rows (source pass), the stage's mask words,
// the mbarriers and the abort flag.
template <int L, bool SRC, bool FR = true>
struct BtcSmem {
  using Sh = BtcShape<L>;
  static constexpr size_t fbuf = 0;
  static constexpr size_t kbuf = fbuf + (FR ? size_t(Sh::STAGES) * Sh::RS * Sh::FSTR : 0);
  static constexpr size_t sbuf = kbuf + size_t(Sh::STAGES) * Sh::RS * kKStr;
  static constexpr size_t mbuf = sbuf + (SRC ? size_t(Sh::STAGES) * Sh::RS * kSStr : 0);
  static constexpr size_t bars = mbuf + size_t(Sh::STAGES) * kTileM * 4;
  static constexpr size_t total = bars + size_t(Sh::STAGES) * 8 + 16;
};

struct BtcParams {
  const __nv_bfloat16* q;   // [n][H][dk]
  const __nv_bfloat16* k;   // [n][H][dk]
  const float* hp;          // h' [n][D][C], values rounded to tf32
  const float* dm;          // dL/dm [n][D][C], float32 (not rounded)
  const int32_t* order;     // tile slot -> atom (null: identity)
  const int* ulen;          // [tiles]
  const int* uni;           // union indices, tile base = toff ? toff[t] : t * cap
  const uint32_t* mask;     // word-major membership words, tile base = base / 2
  const int* toff;          // [tiles + 1] or null
  int cap, tiles;
  float* stats;             // [n][2][H]: lse (read), Delta (target pass writes)
  float* dq;                // [n][H][dk]   target pass
  float* dk;                // [n][H][dk]   source pass
  float* dhp;               // [n][D][C]    source pass
  float* m;                 // [n][D][C]    statistics pass
  int n;
  float qscale;             // log2(e) / sqrt(dk)
  float kscale;             // 1 / sqrt(dk)
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
// D += A B, m16n8k16, bf16 in, f32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D += A B, m16n8k8, tf32 in, f32 accumulate.  Fragments (g = lane / 4,
// t = lane % 4): a0 = A[g][t], a1 = A[g+8][t], a2 = A[g][t+4], a3 = A[g+8][t+4];
// b0 = B[t][g], b1 = B[t+4][g]; d0, d1 = D[g][2t, 2t+1], d2, d3 = D[g+8][2t, 2t+1].
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// float -> tf32, round to nearest (ties away), as a 32-bit pattern
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
  return r;
}
// a bf16 in shared memory as the bit pattern of the equal float (exact in tf32)
__device__ __forceinline__ uint32_t bf16_bits_f32(const unsigned char* p) {
  return uint32_t(*reinterpret_cast<const unsigned short*>(p)) << 16;
}

// The head's 16 key (or query) columns of a stage's staged rows as mma B
// fragments: {b0, b1} of n8 tile 0 in f[0], f[1] and, with 16 rows, of n8
// tile 1 in f[2], f[3].
template <int RS>
__device__ __forceinline__ void stage_frags(uint32_t (&f)[4], const unsigned char* kb, int lane, int h) {
  if constexpr (RS == 16) {
    ldsm_x4(f, smem_u32(kb + ((lane & 7) + 8 * (lane >> 4)) * kKStr + h * 32 + ((lane >> 3) & 1) * 16));
  } else {
    static_assert(RS == 8, "stages of one or two n8 tiles");
    uint32_t r[2];
    ldsm_x2(r, smem_u32(kb + (lane & 7) * kKStr + h * 32 + ((lane >> 3) & 1) * 16));
    f[0] = r[0];
    f[1] = r[1];
    f[2] = f[3] = 0u;
  }
}

// The accumulator fragment of an n8 tile (columns 2t, 2t+1 of rows g, g+8)
// as the A fragment of an m16n8k8 tf32 product whose k index runs over the
// same 8 columns in the order (0, 2, 4, 6, 1, 3, 5, 7): k position t is
// column 2t and k position t + 4 is column 2t + 1, so the B fragment takes
// rows 2t and 2t + 1 of the streamed operand.
__device__ __forceinline__ void acc_as_a(uint32_t (&a)[4], const float (&c)[4]) {
  a[0] = to_tf32(c[0]);
  a[1] = to_tf32(c[2]);
  a[2] = to_tf32(c[1]);
  a[3] = to_tf32(c[3]);
}
// The same as a pair (hi, lo) with hi + lo = c to about 2^-21 relative (lo
// left as float32 bits, which the product truncates to tf32): two tf32
// products then carry c at nearly float32 precision.
__device__ __forceinline__ void acc_as_a_split(uint32_t (&hi)[4], uint32_t (&lo)[4], const float (&c)[4]) {
  acc_as_a(hi, c);
  lo[0] = __float_as_uint(c[0] - __uint_as_float(hi[0]));
  lo[1] = __float_as_uint(c[2] - __uint_as_float(hi[1]));
  lo[2] = __float_as_uint(c[1] - __uint_as_float(hi[2]));
  lo[3] = __float_as_uint(c[3] - __uint_as_float(hi[3]));
}

__device__ __forceinline__ int slot_atom(const int32_t* order, int tile, int r, int n) {
  const long long slot = (long long)tile * kTileM + r;
  if (slot >= n) return -1;
  const int a = order ? order[slot] : int(slot);
  return (unsigned)a < (unsigned)n ? a : -1;
}

// The per-CTA streaming machinery of the passes: the tile's union in stages
// of RS rows; thread r < RS stages row r of each stage (its index loaded one
// stage ahead): its float row (FR), q or k row and (source pass) statistics
// row; thread 0 also the stage's 16 mask words.
template <int L, bool SRC, bool FR = true>
struct Stream {
  using Sh = BtcShape<L>;
  using Sm = BtcSmem<L, SRC, FR>;
  static constexpr int RS = Sh::RS, STAGES = Sh::STAGES, FROW = Sh::FROW, FSTR = Sh::FSTR;
  static_assert(FROW % 16 == 0 && FSTR % 16 == 0, "bulk copies move 16-byte units");
  unsigned char* smem;
  const char* fsrc;        // float rows (h' in the target pass, dm in the source pass)
  const char* ksrc;        // q / k rows
  const char* ssrc;        // stats rows (source pass)
  const uint32_t* mtile;   // the tile's mask words
  const int* utile;        // the tile's union indices
  int n, nst;
  volatile int* abort_flag;

  __device__ uint64_t* bars() const { return reinterpret_cast<uint64_t*>(smem + Sm::bars); }
  __device__ int load_index(int s, int r) const {
    if (s >= nst) return 0;
    const int a = __ldg(utile + s * RS + r);
    return (unsigned)a < (unsigned)n ? a : 0;
  }
  // thread r < RS: row r of stage s (atom a)
  __device__ void issue(int s, int r, int a) const {
    const int buf = s % STAGES;
    const uint32_t bar = smem_u32(bars() + buf);
    const uint32_t bytes = (FR ? FROW : 0) + kKRow + (SRC ? kSRow : 0) + (r == 0 ? kTileM * 4 : 0);
    mbar_arrive_expect_tx(bar, bytes);
    if constexpr (FR)
      bulk_g2s(smem_u32(smem + Sm::fbuf + (size_t(buf) * RS + r) * FSTR), fsrc + (size_t)a * FROW, FROW,
               bar);
    bulk_g2s(smem_u32(smem + Sm::kbuf + (size_t(buf) * RS + r) * kKStr), ksrc + (size_t)a * kKRow,
             kKRow, bar);
    if constexpr (SRC)
      bulk_g2s(smem_u32(smem + Sm::sbuf + (size_t(buf) * RS + r) * kSStr), ssrc + (size_t)a * kSRow,
               kSRow, bar);
    if (r == 0)
      bulk_g2s(smem_u32(smem + Sm::mbuf + size_t(buf) * kTileM * 4), mtile + ((s * RS) >> 5) * kTileM,
               kTileM * 4, bar);
  }
  __device__ void wait(int s) const {
    bounded_wait(smem_u32(bars() + s % STAGES), uint32_t(s / STAGES) & 1u, kWaitPolls, abort_flag);
  }
  // after the loop: if a wait gave up, give the last phase of every buffer a
  // short, bounded chance to land before shared memory is released
  __device__ void drain(int tid) const {
    if (!*abort_flag || tid != 0) return;
    volatile int none = 0;
    for (int b = 0; b < STAGES && b < nst; ++b) {
      const int last = b + (nst - 1 - b) / STAGES * STAGES;
      bounded_wait(smem_u32(bars() + b), uint32_t(last / STAGES) & 1u, kDrainPolls, &none);
    }
  }
};

// Set up a CTA's stream for tile `tile` and start its first STAGES - 1
// stages; returns the index thread r (< RS) stages next.
template <int L, bool SRC, bool FR = true>
__device__ __forceinline__ int stream_begin(Stream<L, SRC, FR>& S, const BtcParams& p, int tile,
                                            unsigned char* smem, int tid) {
  using Sh = BtcShape<L>;
  using Sm = BtcSmem<L, SRC, FR>;
  constexpr int RS = Sh::RS, STAGES = Sh::STAGES;
  const long long base = p.toff ? (long long)p.toff[tile] : (long long)tile * p.cap;
  const int capt = p.toff ? p.toff[tile + 1] - p.toff[tile] : p.cap;
  int U = p.ulen[tile];
  U = U < 0 ? 0 : (U > capt ? capt : U);
  S.smem = smem;
  S.utile = p.uni + base;
  S.mtile = p.mask + base / 2;
  S.n = p.n;
  S.nst = (U + RS - 1) / RS;
  S.abort_flag = reinterpret_cast<volatile int*>(smem + Sm::bars + STAGES * 8);
  if (tid == 0) {
    for (int b = 0; b < STAGES; ++b) mbar_init(smem_u32(S.bars() + b), RS);
    mbar_fence_init();
    *S.abort_flag = 0;
  }
  __syncthreads();
  int nidx = 0;
  if (tid < RS) {
    for (int s = 0; s < STAGES - 1 && s < S.nst; ++s) S.issue(s, tid, S.load_index(s, tid));
    nidx = S.load_index(STAGES - 1, tid);
  }
  return nidx;
}

// ---------------------------------------------------------------- statistics pass
// m_i = sum_j alpha_ij h'_j (WITH_M: only dL/dr needs it) and lse_i per head,
// with the forward kernel's lazy online softmax: a per-row reference maximum
// raised only when a logit exceeds it by more than 2^8 (tested once per
// stage), the accumulators and the weight sums rescaled then.  Without m the
// pass streams the key rows alone.
template <int L, bool WITH_M>
__global__ void __launch_bounds__(kBThreads, 1) bwd_stats_tc_kernel(const __grid_constant__ BtcParams p) {
  using Sh = BtcShape<L>;
  using Sm = BtcSmem<L, false, WITH_M>;
  constexpr int D = Sh::D, RS = Sh::RS, STAGES = Sh::STAGES, FSTR = Sh::FSTR;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, h = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;

  Stream<L, false, WITH_M> S;
  S.fsrc = reinterpret_cast<const char*>(p.hp);
  S.ksrc = reinterpret_cast<const char*>(p.k);
  S.ssrc = nullptr;
  int nidx = stream_begin<L, false, WITH_M>(S, p, tile, smem, tid);

  const int tg0 = slot_atom(p.order, tile, g, p.n), tg1 = slot_atom(p.order, tile, g + 8, p.n);
  uint32_t qa[4];
  {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
    qa[0] = tg0 >= 0 ? __ldg(q32 + (size_t)tg0 * (kBH * 8) + h * 8 + t) : 0u;
    qa[1] = tg1 >= 0 ? __ldg(q32 + (size_t)tg1 * (kBH * 8) + h * 8 + t) : 0u;
    qa[2] = tg0 >= 0 ? __ldg(q32 + (size_t)tg0 * (kBH * 8) + h * 8 + 4 + t) : 0u;
    qa[3] = tg1 >= 0 ? __ldg(q32 + (size_t)tg1 * (kBH * 8) + h * 8 + 4 + t) : 0u;
  }
  const float qs = p.qscale;
  const float inv_qs = 1.f / qs;
  constexpr float kNone = -1e30f;   // finite: a masked logit (-inf) gives exp2(-inf) = 0
  constexpr float kLazy = 8.f;
  float mref0 = kNone, mref1 = kNone;          // log2-domain references of rows g, g+8
  float thr0 = -INFINITY, thr1 = -INFINITY;    // raw-logit thresholds that trigger a raise
  float z0 = 0.f, z1 = 0.f;                    // weight sums (this lane's columns)
  float acc[D][4];
#pragma unroll
  for (int d = 0; d < D; ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[d][e] = 0.f;

  for (int st = 0; st < S.nst; ++st) {
    __syncthreads();
    if (tid < RS && st + STAGES - 1 < S.nst) {
      S.issue(st + STAGES - 1, tid, nidx);
      nidx = S.load_index(st + STAGES, tid);
    }
    S.wait(st);
    const int buf = st % STAGES;
    const unsigned char* fb = smem + Sm::fbuf + size_t(buf) * RS * FSTR;
    const unsigned char* kb = smem + Sm::kbuf + size_t(buf) * RS * kKStr;
    const uint32_t* mw = reinterpret_cast<const uint32_t*>(smem + Sm::mbuf) + buf * kTileM;
    const int sh = (st * RS) & 31;
    const uint32_t m0 = mw[g] >> sh, m1 = mw[g + 8] >> sh;
    uint32_t kf[4];
    stage_frags<RS>(kf, kb, lane, h);
    float v[RS / 8][4];   // masked raw logits: rows g (0, 1), g+8 (2, 3); columns 2t, 2t+1
    bool over = false;
#pragma unroll
    for (int nt = 0; nt < RS / 8; ++nt) {
      float sv[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(sv, qa, kf[2 * nt], kf[2 * nt + 1]);
      const uint32_t w0 = m0 >> (8 * nt + 2 * t), w1 = m1 >> (8 * nt + 2 * t);
      v[nt][0] = (w0 & 1u) ? sv[0] : -INFINITY;
      v[nt][1] = (w0 & 2u) ? sv[1] : -INFINITY;
      v[nt][2] = (w1 & 1u) ? sv[2] : -INFINITY;
      v[nt][3] = (w1 & 2u) ? sv[3] : -INFINITY;
      over |= (v[nt][0] > thr0) | (v[nt][1] > thr0) | (v[nt][2] > thr1) | (v[nt][3] > thr1);
    }
    if (__any_sync(0xffffffffu, over)) {
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < RS / 8; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(v[nt][0], v[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(v[nt][2], v[nt][3]));
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
      z0 *= sc0;
      z1 *= sc1;
      if constexpr (WITH_M) {
#pragma unroll
        for (int d = 0; d < D; ++d) {
          acc[d][0] *= sc0;
          acc[d][1] *= sc0;
          acc[d][2] *= sc1;
          acc[d][3] *= sc1;
        }
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
    for (int nt = 0; nt < RS / 8; ++nt) {
      float P[4];
      P[0] = fast_exp2(fmaf(v[nt][0], qs, -mref0));
      P[1] = fast_exp2(fmaf(v[nt][1], qs, -mref0));
      P[2] = fast_exp2(fmaf(v[nt][2], qs, -mref1));
      P[3] = fast_exp2(fmaf(v[nt][3], qs, -mref1));
      z0 += P[0] + P[1];
      z1 += P[2] + P[3];
      if constexpr (WITH_M) {
        uint32_t pa[4];
        acc_as_a(pa, P);
        // m += P H' (B rows: union atoms 8 nt + 2t, + 1; columns: the head's channels)
        const uint32_t* h0 = reinterpret_cast<const uint32_t*>(fb + (8 * nt + 2 * t) * FSTR) + h * 8 + g;
        const uint32_t* h1 = h0 + FSTR / 4;
#pragma unroll
        for (int d = 0; d < D; ++d) mma_tf32(acc[d], pa, h0[d * kBC], h1[d * kBC]);
      }
    }
  }
  S.drain(tid);

  z0 += __shfl_xor_sync(0xffffffffu, z0, 1);
  z0 += __shfl_xor_sync(0xffffffffu, z0, 2);
  z1 += __shfl_xor_sync(0xffffffffu, z1, 1);
  z1 += __shfl_xor_sync(0xffffffffu, z1, 2);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int tg = half ? tg1 : tg0;
    if (tg < 0) continue;
    const float z = half ? z1 : z0;
    if constexpr (WITH_M) {
      const float inv = z > 0.f ? 1.f / z : 0.f;
      float* o = p.m + (size_t)tg * D * kBC + h * 8 + 2 * t;
#pragma unroll
      for (int d = 0; d < D; ++d)
        *reinterpret_cast<float2*>(o + d * kBC) =
            make_float2(acc[d][2 * half] * inv, acc[d][2 * half + 1] * inv);
    }
    if (t == 0)
      p.stats[(size_t)tg * (2 * kBH) + h] = z > 0.f ? (half ? mref1 : mref0) + __log2f(z) : -INFINITY;
  }
}

// ---------------------------------------------------------------- target pass
template <int L>
__global__ void __launch_bounds__(kBThreads, 1) bwd_target_tc_kernel(const __grid_constant__ BtcParams p) {
  using Sh = BtcShape<L>;
  using Sm = BtcSmem<L, false>;
  constexpr int D = Sh::D, RS = Sh::RS, STAGES = Sh::STAGES, FSTR = Sh::FSTR;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, h = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;

  Stream<L, false> S;
  S.fsrc = reinterpret_cast<const char*>(p.hp);
  S.ksrc = reinterpret_cast<const char*>(p.k);
  S.ssrc = nullptr;
  int nidx = stream_begin<L, false>(S, p, tile, smem, tid);

  // the tile's operands: q (bf16 A fragment of S = Q K^T), dm (tf32 A
  // fragments of dalpha = dm H'^T, one per component), lse of rows g, g+8
  const int tg0 = slot_atom(p.order, tile, g, p.n), tg1 = slot_atom(p.order, tile, g + 8, p.n);
  uint32_t qa[4];
  {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
    qa[0] = tg0 >= 0 ? __ldg(q32 + (size_t)tg0 * (kBH * 8) + h * 8 + t) : 0u;
    qa[1] = tg1 >= 0 ? __ldg(q32 + (size_t)tg1 * (kBH * 8) + h * 8 + t) : 0u;
    qa[2] = tg0 >= 0 ? __ldg(q32 + (size_t)tg0 * (kBH * 8) + h * 8 + 4 + t) : 0u;
    qa[3] = tg1 >= 0 ? __ldg(q32 + (size_t)tg1 * (kBH * 8) + h * 8 + 4 + t) : 0u;
  }
  uint32_t dma[D][4];
  {
    const uint32_t* d32 = reinterpret_cast<const uint32_t*>(p.dm);
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const size_t o = size_t(d) * kBC + h * 8 + t;
      // dm is float32 in memory (the source pass splits it into hi + lo);
      // this pass's products take it rounded to tf32
      dma[d][0] = tg0 >= 0 ? to_tf32(__uint_as_float(__ldg(d32 + (size_t)tg0 * D * kBC + o))) : 0u;
      dma[d][1] = tg1 >= 0 ? to_tf32(__uint_as_float(__ldg(d32 + (size_t)tg1 * D * kBC + o))) : 0u;
      dma[d][2] = tg0 >= 0 ? to_tf32(__uint_as_float(__ldg(d32 + (size_t)tg0 * D * kBC + o + 4))) : 0u;
      dma[d][3] = tg1 >= 0 ? to_tf32(__uint_as_float(__ldg(d32 + (size_t)tg1 * D * kBC + o + 4))) : 0u;
    }
  }
  const float lse0 = tg0 >= 0 ? __ldg(p.stats + (size_t)tg0 * (2 * kBH) + h) : 0.f;
  const float lse1 = tg1 >= 0 ? __ldg(p.stats + (size_t)tg1 * (2 * kBH) + h) : 0.f;
  const float qs = p.qscale;

  float accA[2][4], accB[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) accA[a][e] = accB[a][e] = 0.f;
  float dl0 = 0.f, dl1 = 0.f;   // Delta partials of rows g, g+8

  for (int st = 0; st < S.nst; ++st) {
    __syncthreads();   // every warp is done with the buffer refilled next
    if (tid < RS && st + STAGES - 1 < S.nst) {
      S.issue(st + STAGES - 1, tid, nidx);
      nidx = S.load_index(st + STAGES, tid);
    }
    S.wait(st);
    const int buf = st % STAGES;
    const unsigned char* fb = smem + Sm::fbuf + size_t(buf) * RS * FSTR;
    const unsigned char* kb = smem + Sm::kbuf + size_t(buf) * RS * kKStr;
    const uint32_t* mw = reinterpret_cast<const uint32_t*>(smem + Sm::mbuf) + buf * kTileM;
    const int sh = (st * RS) & 31;
    const uint32_t m0 = mw[g] >> sh, m1 = mw[g + 8] >> sh;
    // key fragments of both n8 tiles of the stage
    uint32_t kf[4];
    stage_frags<RS>(kf, kb, lane, h);
#pragma unroll
    for (int nt = 0; nt < RS / 8; ++nt) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(s, qa, kf[2 * nt], kf[2 * nt + 1]);
      const uint32_t w0 = m0 >> (8 * nt + 2 * t), w1 = m1 >> (8 * nt + 2 * t);
      float P[4];
      P[0] = (w0 & 1u) ? fast_exp2(fmaf(s[0], qs, -lse0)) : 0.f;
      P[1] = (w0 & 2u) ? fast_exp2(fmaf(s[1], qs, -lse0)) : 0.f;
      P[2] = (w1 & 1u) ? fast_exp2(fmaf(s[2], qs, -lse1)) : 0.f;
      P[3] = (w1 & 2u) ? fast_exp2(fmaf(s[3], qs, -lse1)) : 0.f;
      // dalpha for the tile's 16 targets x these 8 union atoms
      float dp[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t hb = smem_u32(fb + (8 * nt + (lane & 7)) * FSTR + h * 32 + ((lane >> 3) & 1) * 16);
      float dp2[4] = {0.f, 0.f, 0.f, 0.f};   // odd components: a second, independent chain
#pragma unroll
      for (int d = 0; d + 1 < D; d += 2) {
        uint32_t r[4];
        ldsm_x4(r, hb + (d + (lane >> 4)) * (kBC * 4));
        mma_tf32(dp, dma[d], r[0], r[1]);
        mma_tf32(dp2, dma[d + 1], r[2], r[3]);
      }
      if constexpr (D % 2) {
        uint32_t r[2];
        ldsm_x2(r, hb + (D - 1) * (kBC * 4));
        mma_tf32(dp, dma[D - 1], r[0], r[1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) dp[e] += dp2[e];
      float E[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) E[e] = P[e] * dp[e];
      dl0 += E[0] + E[1];
      dl1 += E[2] + E[3];
      // A += E K, B += P K over these 8 union atoms (rows 2t, 2t+1 of the
      // n8 tile for k positions t, t+4).  dq = A - Delta B cancels (exactly,
      // for a target with a single neighbour), so E and P enter as hi + lo
      // pairs and A, B keep float32 precision.
      uint32_t ea[4], el[4], pa[4], pl[4];
      acc_as_a_split(ea, el, E);
      acc_as_a_split(pa, pl, P);
      const unsigned char* k0 = kb + (8 * nt + 2 * t) * kKStr + h * 32;
#pragma unroll
      for (int nd = 0; nd < 2; ++nd) {
        const uint32_t b0 = bf16_bits_f32(k0 + (8 * nd + g) * 2);
        const uint32_t b1 = bf16_bits_f32(k0 + kKStr + (8 * nd + g) * 2);
        mma_tf32(accA[nd], ea, b0, b1);
        mma_tf32(accA[nd], el, b0, b1);
        mma_tf32(accB[nd], pa, b0, b1);
        mma_tf32(accB[nd], pl, b0, b1);
      }
    }
  }
  S.drain(tid);

  dl0 += __shfl_xor_sync(0xffffffffu, dl0, 1);
  dl0 += __shfl_xor_sync(0xffffffffu, dl0, 2);
  dl1 += __shfl_xor_sync(0xffffffffu, dl1, 1);
  dl1 += __shfl_xor_sync(0xffffffffu, dl1, 2);
  const float ks = p.kscale;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int tg = half ? tg1 : tg0;
    if (tg < 0) continue;
    const float dl = half ? dl1 : dl0;
    float* o = p.dq + (size_t)tg * (kBH * 16) + h * 16 + 2 * t;
#pragma unroll
    for (int nd = 0; nd < 2; ++nd)
      *reinterpret_cast<float2*>(o + 8 * nd) =
          make_float2((accA[nd][2 * half] - dl * accB[nd][2 * half]) * ks,
                      (accA[nd][2 * half + 1] - dl * accB[nd][2 * half + 1]) * ks);
    if (t == 0) p.stats[(size_t)tg * (2 * kBH) + kBH + h] = dl;
  }
}

// ---------------------------------------------------------------- source pass
// PART selects what one sweep accumulates: kSrcBoth dk and dh' (lmax <= 2);
// at lmax 3 the register-resident h' operand (dk) and dh' accumulator would
// not fit together, so the union is swept twice, kSrcDk then kSrcDh.
enum SourcePart { kSrcBoth, kSrcDk, kSrcDh };
template <int L, int PART>
__global__ void __launch_bounds__(kBThreads, 1) bwd_source_tc_kernel(const __grid_constant__ BtcParams p) {
  constexpr bool DK = PART != kSrcDh, DH = PART != kSrcDk;
  using Sh = BtcShape<L>;
  using Sm = BtcSmem<L, true>;
  constexpr int D = Sh::D, RS = Sh::RS, STAGES = Sh::STAGES, FSTR = Sh::FSTR;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, h = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;

  Stream<L, true> S;
  S.fsrc = reinterpret_cast<const char*>(p.dm);
  S.ksrc = reinterpret_cast<const char*>(p.q);
  S.ssrc = reinterpret_cast<const char*>(p.stats);
  int nidx = stream_begin<L, true>(S, p, tile, smem, tid);

  // the tile's operands: k of the 16 sources (bf16 A fragment of S^T = K Q^T)
  // and h' (tf32 A fragments of dalpha^T = H' dm^T)
  const int sa0 = slot_atom(p.order, tile, g, p.n), sa1 = slot_atom(p.order, tile, g + 8, p.n);
  uint32_t ka[4];
  {
    const uint32_t* k32 = reinterpret_cast<const uint32_t*>(p.k);
    ka[0] = sa0 >= 0 ? __ldg(k32 + (size_t)sa0 * (kBH * 8) + h * 8 + t) : 0u;
    ka[1] = sa1 >= 0 ? __ldg(k32 + (size_t)sa1 * (kBH * 8) + h * 8 + t) : 0u;
    ka[2] = sa0 >= 0 ? __ldg(k32 + (size_t)sa0 * (kBH * 8) + h * 8 + 4 + t) : 0u;
    ka[3] = sa1 >= 0 ? __ldg(k32 + (size_t)sa1 * (kBH * 8) + h * 8 + 4 + t) : 0u;
  }
  uint32_t ha[DK ? D : 1][4];
  if constexpr (DK) {
    const uint32_t* h32 = reinterpret_cast<const uint32_t*>(p.hp);
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const size_t o = size_t(d) * kBC + h * 8 + t;
      ha[d][0] = sa0 >= 0 ? __ldg(h32 + (size_t)sa0 * D * kBC + o) : 0u;
      ha[d][1] = sa1 >= 0 ? __ldg(h32 + (size_t)sa1 * D * kBC + o) : 0u;
      ha[d][2] = sa0 >= 0 ? __ldg(h32 + (size_t)sa0 * D * kBC + o + 4) : 0u;
      ha[d][3] = sa1 >= 0 ? __ldg(h32 + (size_t)sa1 * D * kBC + o + 4) : 0u;
    }
  }
  const float qs = p.qscale;

  float dka[2][4], dha[DH ? D : 1][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) dka[a][e] = 0.f;
#pragma unroll
  for (int d = 0; d < (DH ? D : 1); ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) dha[d][e] = 0.f;

  for (int st = 0; st < S.nst; ++st) {
    __syncthreads();
    if (tid < RS && st + STAGES - 1 < S.nst) {
      S.issue(st + STAGES - 1, tid, nidx);
      nidx = S.load_index(st + STAGES, tid);
    }
    S.wait(st);
    const int buf = st % STAGES;
    const unsigned char* fb = smem + Sm::fbuf + size_t(buf) * RS * FSTR;
    const unsigned char* qb = smem + Sm::kbuf + size_t(buf) * RS * kKStr;
    const unsigned char* sb = smem + Sm::sbuf + size_t(buf) * RS * kSStr;
    const uint32_t* mw = reinterpret_cast<const uint32_t*>(smem + Sm::mbuf) + buf * kTileM;
    const int sh = (st * RS) & 31;
    const uint32_t m0 = mw[g] >> sh, m1 = mw[g + 8] >> sh;
    uint32_t qf[4];
    stage_frags<RS>(qf, qb, lane, h);
#pragma unroll
    for (int nt = 0; nt < RS / 8; ++nt) {
      // rows: sources g, g+8; columns: union targets ca = 8 nt + 2t, cb = ca + 1
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(s, ka, qf[2 * nt], qf[2 * nt + 1]);
      const float* sta = reinterpret_cast<const float*>(sb + (8 * nt + 2 * t) * kSStr);
      const float* stb = reinterpret_cast<const float*>(sb + (8 * nt + 2 * t + 1) * kSStr);
      const float lsa = sta[h], lsb = stb[h], dla = sta[kBH + h], dlb = stb[kBH + h];
      const uint32_t w0 = m0 >> (8 * nt + 2 * t), w1 = m1 >> (8 * nt + 2 * t);
      float P[4];
      P[0] = (w0 & 1u) ? fast_exp2(fmaf(s[0], qs, -lsa)) : 0.f;
      P[1] = (w0 & 2u) ? fast_exp2(fmaf(s[1], qs, -lsb)) : 0.f;
      P[2] = (w1 & 1u) ? fast_exp2(fmaf(s[2], qs, -lsa)) : 0.f;
      P[3] = (w1 & 2u) ? fast_exp2(fmaf(s[3], qs, -lsb)) : 0.f;
      if constexpr (DK) {
      float dp[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t db = smem_u32(fb + (8 * nt + (lane & 7)) * FSTR + h * 32 + ((lane >> 3) & 1) * 16);
      float dp2[4] = {0.f, 0.f, 0.f, 0.f};   // odd components: a second, independent chain
      // dm rows are float32: rounded to tf32 here (the tensor core would
      // truncate them, which doubles the error dk inherits from dalpha)
#pragma unroll
      for (int d = 0; d + 1 < D; d += 2) {
        uint32_t r[4];
        ldsm_x4(r, db + (d + (lane >> 4)) * (kBC * 4));
        mma_tf32(dp, ha[d], to_tf32(__uint_as_float(r[0])), to_tf32(__uint_as_float(r[1])));
        mma_tf32(dp2, ha[d + 1], to_tf32(__uint_as_float(r[2])), to_tf32(__uint_as_float(r[3])));
      }
      if constexpr (D % 2) {
        uint32_t r[2];
        ldsm_x2(r, db + (D - 1) * (kBC * 4));
        mma_tf32(dp, ha[D - 1], to_tf32(__uint_as_float(r[0])), to_tf32(__uint_as_float(r[1])));
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) dp[e] += dp2[e];
      float ds[4];
      ds[0] = P[0] * (dp[0] - dla);
      ds[1] = P[1] * (dp[1] - dlb);
      ds[2] = P[2] * (dp[2] - dla);
      ds[3] = P[3] * (dp[3] - dlb);
      uint32_t dsa[4];
      acc_as_a(dsa, ds);
      // dk += ds^T Q (B rows: union targets ca, cb)
      const unsigned char* q0 = qb + (8 * nt + 2 * t) * kKStr + h * 32;
#pragma unroll
      for (int nd = 0; nd < 2; ++nd)
        mma_tf32(dka[nd], dsa, bf16_bits_f32(q0 + (8 * nd + g) * 2),
                 bf16_bits_f32(q0 + kKStr + (8 * nd + g) * 2));
      }
      if constexpr (DH) {
      uint32_t pa[4], pl[4];
      acc_as_a_split(pa, pl, P);
      // dh' += alpha^T dm (B rows: dm of ca, cb; columns: the head's channels)
      // in three tf32 products of the hi/lo splits of both operands,
      // alpha_hi dm_hi + alpha_lo dm_hi + alpha_hi dm_lo: float32-level
      // accuracy, which the adjoint source coupling needs (its |r|^l-scaled
      // terms cancel on small channels of dL/dh)
      // (hi = dm rounded to tf32; lo = dm - hi, which the product truncates to
      // tf32: its error is 2^-10 of lo, about 2^-21 of dm).  Components go in
      // pairs, so no product waits on the one just issued into its accumulator.
      const float* d0 = reinterpret_cast<const float*>(fb + (8 * nt + 2 * t) * FSTR) + h * 8 + g;
      const float* d1 = d0 + FSTR / 4;
      auto split = [](float x, uint32_t& hi, uint32_t& lo) {
        hi = to_tf32(x);
        lo = __float_as_uint(x - __uint_as_float(hi));
      };
#pragma unroll
      for (int d = 0; d < D; d += 2) {
        constexpr int kLast = D - 1;
        const int e = d + 1 <= kLast ? d + 1 : kLast;
        uint32_t ha0, ha1, la0, la1, hb0, hb1, lb0, lb1;
        split(d0[d * kBC], ha0, la0);
        split(d1[d * kBC], ha1, la1);
        split(d0[e * kBC], hb0, lb0);
        split(d1[e * kBC], hb1, lb1);
        mma_tf32(dha[d], pa, ha0, ha1);
        if (e != d) mma_tf32(dha[e], pa, hb0, hb1);
        mma_tf32(dha[d], pl, ha0, ha1);
        if (e != d) mma_tf32(dha[e], pl, hb0, hb1);
        mma_tf32(dha[d], pa, la0, la1);
        if (e != d) mma_tf32(dha[e], pa, lb0, lb1);
      }
      }
    }
  }
  S.drain(tid);

  const float ks = p.kscale;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int sa = half ? sa1 : sa0;
    if (sa < 0) continue;
    if constexpr (DK) {
      float* o = p.dk + (size_t)sa * (kBH * 16) + h * 16 + 2 * t;
#pragma unroll
      for (int nd = 0; nd < 2; ++nd)
        *reinterpret_cast<float2*>(o + 8 * nd) =
            make_float2(dka[nd][2 * half] * ks, dka[nd][2 * half + 1] * ks);
    }
    if constexpr (DH) {
      float* od = p.dhp + (size_t)sa * D * kBC + h * 8 + 2 * t;
#pragma unroll
      for (int d = 0; d < D; ++d)
        *reinterpret_cast<float2*>(od + d * kBC) = make_float2(dha[d][2 * half], dha[d][2 * half + 1]);
    }
  }
}

// ---------------------------------------------------------------- plans
// Per source tile: the capacity of its union (the sum of its sources'
// in-degrees, rounded up to a multiple of kPlanPad, at least one pad).
__global__ void csr_tile_cap_kernel(const int* __restrict__ ptr, const int32_t* __restrict__ order, int n,
                                    int tiles, int* __restrict__ capv) {
  const int tl = blockIdx.x * blockDim.x + threadIdx.x;
  if (tl >= tiles) return;
  long long s = 0;
  for (int r = 0; r < kTileM; ++r) {
    const int a = slot_atom(order, tl, r, n);
    if (a >= 0) s += ptr[a + 1] - ptr[a];
  }
  const long long c = (s + kPlanPad - 1) / kPlanPad * kPlanPad;
  capv[tl] = int(c > kPlanPad ? c : kPlanPad);
}

constexpr int kCsrPlanThreads = 256;
struct CsrPlanParams {
  const int* ptr;          // [n + 1] row offsets of the in-lists
  const int* col;          // in-list entries (targets)
  const int32_t* order;
  const int* toff;         // [tiles + 1]
  int* ulen;
  int* uni;
  uint32_t* mask;
  int n, tiles;
};

// One CTA per source tile: the union of its sources' in-lists from a bitmap
// over all atoms (ascending atom index), padded with a valid index whose mask
// bits stay zero, and one membership bit per (source, target) in the
// word-major layout of the forward plan, at the tile's own offset.
__global__ void __launch_bounds__(kCsrPlanThreads) build_csr_plan_kernel(const __grid_constant__ CsrPlanParams p) {
  extern __shared__ uint32_t sm[];
  const int nw = (p.n + 31) / 32;
  uint32_t* bitmap = sm;
  uint32_t* prefix = sm + nw;
  __shared__ int rbeg[kTileM], rlen[kTileM];
  __shared__ int warp_sum[kCsrPlanThreads / 32];
  __shared__ int s_unique;
  const int tile = blockIdx.x;
  const long long base = p.toff[tile];
  const int capt = p.toff[tile + 1] - p.toff[tile];
  uint32_t* gmask = p.mask + base / 2;
  if (threadIdx.x < kTileM) {
    const int a = slot_atom(p.order, tile, threadIdx.x, p.n);
    rbeg[threadIdx.x] = a >= 0 ? p.ptr[a] : 0;
    rlen[threadIdx.x] = a >= 0 ? p.ptr[a + 1] - p.ptr[a] : 0;
  }
  for (int i = threadIdx.x; i < nw; i += blockDim.x) bitmap[i] = 0u;
  for (int i = threadIdx.x; i < capt / 2; i += blockDim.x) gmask[i] = 0u;
  __syncthreads();
  auto for_each_entry = [&](auto&& f) {
    for (int r = 0; r < kTileM; ++r) {
      const int* row = p.col + rbeg[r];
      for (int e = threadIdx.x; e < rlen[r]; e += blockDim.x) f(r, row[e]);
    }
  };
  for_each_entry([&](int, int j) {
    if ((unsigned)j < (unsigned)p.n) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
  });
  __syncthreads();
  const int per = (nw + kCsrPlanThreads - 1) / kCsrPlanThreads;
  const int w0 = threadIdx.x * per;
  const int w1 = min(w0 + per, nw);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bitmap[w]);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[wid] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int w = 0; w < kCsrPlanThreads / 32; ++w) {
      const int v = warp_sum[w];
      warp_sum[w] = acc;
      acc += v;
    }
    s_unique = acc;
  }
  __syncthreads();
  const int U = s_unique < capt ? s_unique : capt;   // never above: U <= sum of the in-degrees
  int* uni = p.uni + base;
  {
    int pos = warp_sum[wid] + incl - mine;
    for (int w = w0; w < w1; ++w) {
      prefix[w] = uint32_t(pos);
      uint32_t b = bitmap[w];
      while (b) {
        const int bit = __ffs(b) - 1;
        if (pos < capt) uni[pos] = w * 32 + bit;
        ++pos;
        b &= b - 1;
      }
    }
  }
  __syncthreads();
  const int upad = U > 0 ? (U + kPlanPad - 1) / kPlanPad * kPlanPad : kPlanPad;
  const int filler = U > 0 ? uni[0] : 0;
  for (int e = U + threadIdx.x; e < upad; e += blockDim.x) uni[e] = filler;
  if (threadIdx.x == 0) p.ulen[tile] = U;
  for_each_entry([&](int r, int j) {
    if ((unsigned)j >= (unsigned)p.n) return;
    const int pos = int(prefix[j >> 5]) + __popc(bitmap[j >> 5] & ((1u << (j & 31)) - 1u));
    if (pos < capt) atomicOr(&gmask[(pos >> 5) * kTileM + r], 1u << (pos & 31));
  });
}

enum PassKind { kStatsPass, kTargetPass, kSourcePass };

template <int L>
int launch_pass_t(const BtcParams& p, PassKind kind, cudaStream_t st) {
  // the statistics pass without m (no dL/dr wanted) streams the key rows alone
  const bool lean = kind == kStatsPass && !p.m;
  const size_t shm = kind == kSourcePass ? BtcSmem<L, true>::total
                     : lean ? BtcSmem<L, false, false>::total : BtcSmem<L, false>::total;
  if (shm > 227 * 1024) return EGAT_ERR_UNSUPPORTED;
  auto run = [&](void (*kern)(BtcParams)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shm)) != cudaSuccess)
      return EGAT_ERR_CUDA;
    kern<<<p.tiles, kBThreads, shm, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
  };
  if (kind == kSourcePass) {
    if constexpr (L >= 3) {
      // two sweeps of the source union: dk, then dh'
      const int e = run(bwd_source_tc_kernel<L, kSrcDk>);
      return e == EGAT_OK ? run(bwd_source_tc_kernel<L, kSrcDh>) : e;
    } else {
      return run(bwd_source_tc_kernel<L, kSrcBoth>);
    }
  }
  auto kern = kind == kTargetPass ? bwd_target_tc_kernel<L>
              : lean ? bwd_stats_tc_kernel<L, false> : bwd_stats_tc_kernel<L, true>;
  return run(kern);
}

int launch_pass(int lmax, const BtcParams& p, PassKind kind, cudaStream_t st) {
  switch (lmax) {
    case 1: return launch_pass_t<1>(p, kind, st);
    case 2: return launch_pass_t<2>(p, kind, st);
    case 3: return launch_pass_t<3>(p, kind, st);
    default: return EGAT_ERR_UNSUPPORTED;
  }
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

bool bwd_tc_supported(const egat_shape& s) {
  static_assert(BtcSmem<1, true>::total <= 227 * 1024 && BtcSmem<2, true>::total <= 227 * 1024 &&
                    BtcSmem<3, true>::total <= 227 * 1024 && BtcSmem<3, false>::total <= 227 * 1024,
                "stages fit the shared memory");
  return s.lmax <= 3 && tc_attention_supported(s) &&
         (long long)s.n * s.K + (long long)kPlanPad * ((s.n + kTileM - 1) / kTileM) < (1LL << 31);
}

size_t bwd_tc_ws_bytes(const egat_shape& s) {
  const size_t n = size_t(s.n), tiles = (n + kTileM - 1) / kTileM;
  const size_t D = size_t(s.lmax + 1) * (s.lmax + 1);
  const size_t ucap = n * s.K + size_t(kPlanPad) * tiles;
  return a256(n * D * s.C * 4)                        // m (float)
         + a256(n * D * s.C * 4)                      // dh' (float)
         + a256(n * 2 * s.H * 4)                      // stats
         + plan_bytes(s.n, s.K, s.lmax)               // forward plan
         + 3 * a256((tiles + 1) * 4)                  // source plan: capacities, offsets, lengths
         + a256(ucap * 4) + a256(ucap / 2 * 4);       // source plan: union, mask
}

BwdTcWs bwd_tc_ws(const egat_shape& s, void* base) {
  const size_t n = size_t(s.n), tiles = (n + kTileM - 1) / kTileM;
  const size_t D = size_t(s.lmax + 1) * (s.lmax + 1);
  const size_t ucap = n * s.K + size_t(kPlanPad) * tiles;
  char* b = static_cast<char*>(base);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    void* ptr = b + o;
    o += a256(bytes);
    return ptr;
  };
  BwdTcWs w;
  w.m = static_cast<float*>(take(n * D * s.C * 4));
  w.dhp = static_cast<float*>(take(n * D * s.C * 4));
  w.stats = static_cast<float*>(take(n * 2 * s.H * 4));
  w.plan = b + o;
  o += plan_bytes(s.n, s.K, s.lmax);
  w.capv = static_cast<int*>(take((tiles + 1) * 4));
  w.toff = static_cast<int*>(take((tiles + 1) * 4));
  w.ulen = static_cast<int*>(take((tiles + 1) * 4));
  w.uni = static_cast<int*>(take(ucap * 4));
  w.mask = static_cast<uint32_t*>(take(ucap / 2 * 4));
  return w;
}

int launch_backward_tc(const egat_shape& s, const BwdTcWs& w, const void* d_q, const void* d_k,
                       const float* d_hp, const float* d_dm, const int32_t* d_order,
                       const int* d_in_ptr, const int* d_in, float* d_dq, float* d_dk, bool want_m,
                       cudaStream_t st) {
  const int tiles = (s.n + kTileM - 1) / kTileM;
  const PlanView fp = plan_view(w.plan, s.n, s.K, s.lmax);
  BtcParams p;
  p.q = static_cast<const __nv_bfloat16*>(d_q);
  p.k = static_cast<const __nv_bfloat16*>(d_k);
  p.hp = d_hp;
  p.dm = d_dm;
  p.order = d_order;
  p.stats = w.stats;
  p.dq = d_dq;
  p.dk = d_dk;
  p.dhp = w.dhp;
  p.m = want_m ? w.m : nullptr;
  p.n = s.n;
  p.qscale = float(1.4426950408889634 / std::sqrt(double(s.dk)));
  p.kscale = float(1.0 / std::sqrt(double(s.dk)));
  // target pass over the forward plan's tiles
  p.ulen = fp.ulen;
  p.uni = fp.uni;
  p.mask = fp.mask;
  p.toff = nullptr;
  p.cap = fp.cap;
  p.tiles = fp.tiles;
  int e = launch_pass(s.lmax, p, kStatsPass, st);
  if (e == EGAT_OK) e = launch_pass(s.lmax, p, kTargetPass, st);
  if (e != EGAT_OK) return e;
  // source plan from the in-lists, then the source pass
  csr_tile_cap_kernel<<<(tiles + 127) / 128, 128, 0, st>>>(d_in_ptr, d_order, s.n, tiles, w.capv);
  if (cudaGetLastError() != cudaSuccess) return EGAT_ERR_CUDA;
  e = launch_exclusive_scan(w.capv, tiles, w.toff, st);
  if (e != EGAT_OK) return e;
  CsrPlanParams cp;
  cp.ptr = d_in_ptr;
  cp.col = d_in;
  cp.order = d_order;
  cp.toff = w.toff;
  cp.ulen = w.ulen;
  cp.uni = w.uni;
  cp.mask = w.mask;
  cp.n = s.n;
  cp.tiles = tiles;
  const size_t shm = 2 * ((size_t(s.n) + 31) / 32) * 4;
  if (shm > kPlanSmemLimit) return EGAT_ERR_UNSUPPORTED;
  if (shm > 48 * 1024 &&
      cudaFuncSetAttribute(build_csr_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(shm)) !=
          cudaSuccess)
    return EGAT_ERR_CUDA;
  build_csr_plan_kernel<<<tiles, kCsrPlanThreads, shm, st>>>(cp);
  if (cudaGetLastError() != cudaSuccess) return EGAT_ERR_CUDA;
  p.ulen = w.ulen;
  p.uni = w.uni;
  p.mask = w.mask;
  p.toff = w.toff;
  p.cap = 0;
  p.tiles = tiles;
  return launch_pass(s.lmax, p, kSourcePass, st);
}

int take_wait_timeouts_backward(cudaStream_t st, unsigned int* count) {
  return take_unit_wait_timeouts(st, count) == 0 ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
