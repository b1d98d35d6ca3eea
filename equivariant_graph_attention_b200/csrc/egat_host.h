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

// Per-tile neighbour union and membership bitmask (device memory views).
struct PlanView {
  int* ulen;        // [tiles] union length
  int* uni;         // [tiles][cap] union atom indices (ascending), padded to kTileK
  uint32_t* mask;   // [tiles][kTileM][cap / 32] bit u of row r: union atom u is a neighbour
  int cap;          // union capacity per tile (power of two >= kTileM * K)
  int tiles;
};
int plan_capacity(int K);
// shared memory of the plan kernel: two bitmap-sized arrays over all atoms and
// one tile mask; the tensor-core path is used while this fits a CTA
size_t plan_smem_bytes(int n, int K);
constexpr size_t kPlanSmemLimit = 200 * 1024;
size_t plan_bytes(int n, int K);
PlanView plan_view(void* base, int n, int K);
int launch_build_plan(int n, int K, const int32_t* d_nbr, const int32_t* d_cnt,
                      const int32_t* d_order, void* d_plan, cudaStream_t st);
// Tiled tensor-core attention (bf16 storage, C/H = 8, dk = 16): fused = true
// applies the target coupling and writes ^h; false writes m.
bool tc_attention_supported(const egat_shape& s);
int launch_attention_tc(const egat_shape& s, bool fused, const void* d_q, const void* d_k,
                        const void* d_hp, const void* d_plan, const int32_t* d_order,
                        const float* d_pos, const float* d_w2, float* d_out, cudaStream_t st);

}  // namespace egat
