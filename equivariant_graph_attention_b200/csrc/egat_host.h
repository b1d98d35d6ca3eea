// Host-side declarations shared by the egat translation units (not part of
// the public ABI; see include/egat.h for that).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "egat.h"

namespace egat {

struct EaasTable;

// Axis-frame re-index factors for every path of degree L ([EX] §2.2): built
// once per L on the host from Clebsch–Gordan coefficients.
const EaasTable& eaas_table(int L);

// Clebsch–Gordan coefficient <j1 m1; j2 m2 | J M> (Racah's formula).
double clebsch_gordan(int j1, int m1, int j2, int m2, int J, int M);

size_t graph_workspace_bytes(int n);
int build_graph(const int32_t* d_pos_q, int n, int cutoff_q, int K, int mode, int32_t* d_a,
                int32_t* d_b, long long col_capacity, int32_t* d_order, int32_t* d_overflow,
                void* d_ws, size_t ws_bytes, cudaStream_t st);

// Step 2 on n atoms: y = EAAS(x, pos, w); x and y in the storage type.
int launch_eaas_source(const egat_shape& s, const void* d_x, const float* d_pos,
                       const float* d_w, void* d_y, cudaStream_t st);

// Step 3 (fused = false: writes m) or steps 3+4 (fused = true: writes ^h).
int launch_attention(const egat_shape& s, bool fused, const void* d_q, const void* d_k,
                     const void* d_hp, const int32_t* d_a, const int32_t* d_b,
                     const int32_t* d_order, const float* d_pos, const float* d_w2,
                     float* d_out, cudaStream_t st);

inline size_t storage_bytes(int dtype) { return dtype == EGAT_BF16 ? 2 : 4; }

// ---- tensor-core attention: tiles of kTileM targets, k-steps of kTileK union atoms
constexpr int kTileM = 16;
constexpr int kTileK = 16;

// Per-tile neighbour union, membership bitmask and target record (device
// memory views).  Unions are padded to whole multiples of kPlanPad entries
// (at least one, also for an empty union) with a valid atom index whose mask
// bits are zero, so that a consumer may stream them in chunks of kPlanPad.
constexpr int kPlanPad = 32;
struct PlanView {
  int* ulen;        // [tiles] union length
  int* uni;         // [tiles][cap] union atom indices (ascending), padded to kPlanPad
  uint32_t* mask;   // [tiles][cap / 32][kTileM] word w of row r: bits of union atoms 32w..32w+31
  float* rec;       // [tiles][plan_record_words(lmax)] target ids, |r|^l, Wigner-D (see below)
  int* sched;       // the attention kernel's tile-claim counter: zeroed by the plan
                    // builder, zero again after every launch
  int cap;          // union capacity per tile (power of two >= kTileM * K)
  int tiles;
};
// Tile record (words): a header (union length, three zeros), int32
// target[kTileM] (-1 past n), float rpow[kTileM][lmax+1] (|r|^0..|r|^lmax),
// float D[kTileM][wig] (real Wigner-D of the alignment rotation, degrees
// 0..lmax, wig = sum of (2l+1)^2) — everything the attention kernel needs per
// tile besides the union itself, so it builds nothing per tile.
constexpr int kRecHdr = 4;
constexpr int rec_wig_size(int lmax) { return (lmax + 1) * (2 * lmax + 1) * (2 * lmax + 3) / 3; }
constexpr int kRecTgt = kRecHdr;
constexpr int kRecRp = kRecHdr + kTileM;
constexpr int rec_off_D(int lmax) { return kRecHdr + kTileM * (2 + lmax); }
constexpr int plan_record_words(int lmax) { return rec_off_D(lmax) + kTileM * rec_wig_size(lmax); }
int plan_capacity(int K);
// shared memory of the plan kernel: two bitmap-sized arrays over all atoms and
// one tile mask; the tensor-core path is used while this fits a CTA
size_t plan_smem_bytes(int n, int K);
constexpr size_t kPlanSmemLimit = 200 * 1024;
size_t plan_bytes(int n, int K, int lmax);
PlanView plan_view(void* base, int n, int K, int lmax);
int launch_build_plan(int n, int K, int lmax, const int32_t* d_nbr, const int32_t* d_cnt,
                      const int32_t* d_order, const float* d_pos, void* d_plan, cudaStream_t st);
// Step 2 with a float32 result whatever the storage type (the per-target
// backward keeps its intermediates in float32).
int launch_eaas_source_f32out(const egat_shape& s, const void* d_x, const float* d_pos,
                              const float* d_w, float* d_y, cudaStream_t st);
// Step 2 for every atom listed in a plan's tile records, rotations from them.
int launch_eaas_planned(const egat_shape& s, const void* d_x, const void* d_plan, const float* d_w,
                        void* d_y, cudaStream_t st);
// The same for bf16 features with C = 128, the result float32 rounded to tf32
// (the backward's operand format).
int launch_eaas_planned_tf32out(const egat_shape& s, const void* d_x, const void* d_plan, const float* d_w,
                                float* d_y, cudaStream_t st);
// Tiled tensor-core attention (bf16 storage, C/H = 8, dk = 16): fused = true
// applies the target coupling and writes ^h; false writes m.
bool tc_attention_supported(const egat_shape& s);
// Backward pass (gradients of <G, ^h> with respect to h, q, k): workspace and launch.
size_t backward_ws_bytes(const egat_shape& s);
int launch_backward(const egat_shape& s, const void* d_h, const float* d_pos, const void* d_q,
                    const void* d_k, const int32_t* d_nbr, const int32_t* d_cnt,
                    const int32_t* d_order, const float* d_w1, const float* d_w2, const float* d_g,
                    void* d_ws, float* d_dh, float* d_dq, float* d_dk, float* d_dpos,
                    cudaStream_t st);
// Exclusive scan of in[0..n) into out[0..n] (out[n] = total) by one CTA.
int launch_exclusive_scan(const int* d_in, int n, int* d_out, cudaStream_t st);
// Tiled tensor-core backward (bf16 storage, C = 128, H = 16, dk = 16,
// lmax <= 2): workspace views and launches.
struct BwdTcWs {
  float* m;        // m [n][D][C] (the statistics pass)
  float* dhp;      // dL/dh' [n][D][C]
  float* stats;    // [n][2][H]: log-sum-exp, Delta
  void* plan;      // forward plan (target tiles)
  int* capv;       // [tiles + 1] source tile capacities
  int* toff;       // [tiles + 1] source tile offsets
  int* ulen;       // [tiles] source tile union lengths
  int* uni;        // source tile unions
  uint32_t* mask;  // source tile membership words
};
bool bwd_tc_supported(const egat_shape& s);
size_t bwd_tc_ws_bytes(const egat_shape& s);
BwdTcWs bwd_tc_ws(const egat_shape& s, void* base);
// m and the log-sum-exp (statistics pass), dq and Delta (target pass), both
// over the forward plan's tiles in w.plan; the source plan from the in-lists,
// dk and dh' (source pass).  d_hp and d_dm float32 rounded to tf32.
// want_m = false (no dL/dr wanted) skips m: the statistics pass streams key rows alone.
int launch_backward_tc(const egat_shape& s, const BwdTcWs& w, const void* d_q, const void* d_k,
                       const float* d_hp, const float* d_dm, const int32_t* d_order,
                       const int* d_in_ptr, const int* d_in, float* d_dq, float* d_dk, bool want_m,
                       cudaStream_t st);
int take_wait_timeouts_backward(cudaStream_t st, unsigned int* count);
// dst[r] = src[idx[r]] for r < count (rows of row_bytes, a multiple of 16; an
// index outside [0, n_src) gives a zero row).
int launch_gather_rows(const void* d_src, long long n_src, long long row_bytes, const int32_t* d_idx,
                       long long count, void* d_dst, cudaStream_t st);
// Bounded-wait reports (one per compilation unit with mbarrier waits): read
// and clear the count of waits that gave up (synchronises st); the self-test
// launch.
int take_wait_timeouts_attention(cudaStream_t st, unsigned int* count);
int take_wait_timeouts_projection(cudaStream_t st, unsigned int* count);
// Edge-centric eSCN convolution (the comparison workload): weights per channel
// and its launch.
int escn_num_weights_host(int lmax, int mmax);
int launch_escn_conv(const egat_shape& s, int mmax, const void* d_h, const float* d_pos,
                     const int32_t* d_nbr, const int32_t* d_cnt, const int32_t* d_order,
                     const float* d_w, float* d_out, cudaStream_t st);
// Invariant query/key projection from the degree-0 channels (tensor cores for
// bf16 storage with C = 128 and H * dk = 256, a plain kernel otherwise).
bool projection_tc_supported(const egat_shape& s);
int launch_qk_projection(const egat_shape& s, const void* d_h, const float* d_wq, const float* d_wk,
                         void* d_q, void* d_k, cudaStream_t st);
int take_wait_timeouts_coupling(cudaStream_t st, unsigned int* count);
int launch_wait_timeout_selftest(int polls, cudaStream_t st);
int launch_attention_tc(const egat_shape& s, bool fused, const void* d_q, const void* d_k,
                        const void* d_hp, const void* d_plan, const float* d_w2, float* d_out,
                        cudaStream_t st);

}  // namespace egat
