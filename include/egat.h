/*
 * egat — equivariant graph attention hot path for NVIDIA B200 (sm_100a).
 *
 * C ABI of the library libegat.so.  Every entry point takes plain pointers and
 * sizes; "d_" pointers are CUDA device pointers, everything else is host
 * memory.  The caller allocates every buffer (inputs, outputs and scratch
 * "workspace", sized by the *_workspace_bytes queries); the library allocates
 * no memory of its own.  All work is enqueued asynchronously on the given
 * stream (a cudaStream_t passed as void*, NULL = legacy default stream); no
 * call synchronises the device.  Calls report errors by return code and never
 * abort, trap or print.
 *
 * Pages cited (by title):
 *  [EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" (explainer)
 *  [TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
 *       Memory" (technical summary)
 *
 * The four steps ([EX] §3.1 node-centric factorisation, [EX] §2 EAAS):
 *  1. egat_build_graph    radius graph from positions (cell list);
 *  2. egat_eaas_couple    h'_j = h_j (x) R(r_j) by EAAS;
 *  3. egat_otf_attention  m_i = sum_j softmax_j(q_i.k_j/sqrt(dk)) h'_j, streamed;
 *  4. egat_otf_attention_coupled  3 with the target coupling ^h_i = m_i (x) R(r_i)
 *                         fused into the attention epilogue;
 *     egat_forward        2 then 3+4.
 *
 * Conventions shared by all calls
 *  - Irrep features are row-major [n][D][C], D = (lmax+1)^2, component index
 *    l*l + l + m (m = -l..l), channel fastest.  Real spherical-harmonic basis
 *    (Condon–Shortley phase cancelled), degree 1 ordered (y, z, x).
 *  - R^l(r) are Racah-normalised solid harmonics of the position vector r as
 *    given (callers centre positions on the system centroid).
 *  - Coupling paths (li, lf, lo) are all triples <= lmax with
 *    |li-lf| <= lo <= li+lf (odd li+lf+lo included), ordered by lo, then li,
 *    then lf ascending; egat_num_paths(lmax) of them (5, 15, 34 for lmax 1-3).
 *    Weights are float32 [P][C]: w[p][c] scales path p of channel c.
 *  - Channel c belongs to head floor(c*H/C); logits are per head.
 *  - Positions for the graph are int32 grid coordinates [n][3]; the float32
 *    positions used for geometry [n][3] must equal them times the grid step
 *    the caller chose (2^-16 Å in this project's inputs).
 *  - Supported shapes: 1 <= lmax <= 3; C in {16, 32, 64, 128}; H a power of
 *    two with C/H a multiple of 8; dk in {8, 16, 32} with H*dk <= 256;
 *    1 <= K <= 1024.  Feature pointers must be 16-byte aligned.
 */
#ifndef EGAT_H
#define EGAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EGAT_VERSION 1

#if defined(__GNUC__)
#define EGAT_API __attribute__((visibility("default")))
#else
#define EGAT_API
#endif

/* return codes: 0 success, negative errors */
enum {
  EGAT_OK = 0,
  EGAT_ERR_ARG = -1,          /* null pointer, bad size or misaligned pointer */
  EGAT_ERR_UNSUPPORTED = -2,  /* shape outside the supported set above */
  EGAT_ERR_CUDA = -3,         /* a CUDA launch or runtime call failed */
  EGAT_ERR_WORKSPACE = -4,    /* workspace smaller than the query returned */
  EGAT_ERR_SCRATCH_LIMIT = -5, /* egat_forward_noalloc: problem larger than its fixed scratch */
  EGAT_ERR_TIMEOUT = -6        /* egat_take_device_status: a bounded device wait gave up */
};

/* storage type of h, q, k and h' (accumulation and outputs are float32) */
enum { EGAT_F32 = 0, EGAT_BF16 = 1 };

/* neighbour-list format */
enum {
  EGAT_GRAPH_PADDED = 0,  /* nbr int32 [n][K] (unused slots -1) + cnt int32 [n] */
  EGAT_GRAPH_CSR = 1      /* rowptr int32 [n+1] + col int32 [n_edges] */
};

typedef struct egat_shape {
  int32_t n;           /* atoms */
  int32_t lmax;        /* highest irrep degree, 1..3 */
  int32_t C;           /* channels per degree */
  int32_t H;           /* attention heads */
  int32_t dk;          /* query/key width per head */
  int32_t K;           /* padded neighbour slots (PADDED) */
  int32_t dtype;       /* EGAT_F32 or EGAT_BF16 */
  int32_t graph_mode;  /* EGAT_GRAPH_PADDED or EGAT_GRAPH_CSR */
  int64_t n_edges;     /* CSR: length of col (row ranges are clamped to it) */
} egat_shape;

/* Library version (EGAT_VERSION). */
EGAT_API int egat_version(void);

/* Static description of a return code. */
EGAT_API const char* egat_strerror(int code);

/* Number of coupling paths P for lmax (0 if lmax is out of range). */
EGAT_API int egat_num_paths(int lmax);

/*
 * Step 1 — radius graph ([EX] §5.1 edge_cutoff, §5.2 neighbour-list check).
 * Atom j != i is a neighbour of i when |p_j - p_i|^2 <= cutoff_q^2, computed
 * exactly in 64-bit integers on grid coordinates (inclusive cutoff).  Cells
 * of edge ceil(cutoff_q / 2) are hashed to a power-of-two table by a Morton
 * code of the cell coordinates, so memory depends only on n, not on the box.
 *
 *  d_pos_q       int32 [n][3] grid coordinates
 *  cutoff_q      cutoff in grid units, > 0
 *  mode          EGAT_GRAPH_PADDED:
 *                  d_nbr_or_rowptr = nbr int32 [n][K]: the neighbours, then
 *                  -1; an atom with more than K keeps the K nearest (ties at
 *                  the K-th distance keep the smaller index);
 *                  d_cnt_or_col = cnt int32 [n] = min(degree, K);
 *                  *d_overflow = number of neighbours dropped.
 *                EGAT_GRAPH_CSR:
 *                  d_nbr_or_rowptr = rowptr int32 [n+1];
 *                  d_cnt_or_col = col int32 [col_capacity]; entries past
 *                  col_capacity are not written and *d_overflow = their
 *                  number.
 *                Row order: cell order of the neighbourhood (atoms of one
 *                cell by index); a truncated padded row lists its K nearest
 *                by (squared distance, index).  Deterministic: the same
 *                arrays on every call.
 *  d_order       optional int32 [n]: atoms listed cell by cell (Morton
 *                order of cells) — a traversal order with spatial locality
 *                for egat_otf_attention / egat_forward.  May be NULL.
 *  d_overflow    int32 [1], zeroed and then set by this call.
 *  d_ws, ws_bytes  scratch of at least egat_graph_workspace_bytes(n).
 * Returns EGAT_ERR_UNSUPPORTED when cutoff_q > 2^26 (1,024 Å on a 2^-16 Å
 * grid) or cutoff_q^2 * 2^ceil(log2 n) >= 2^64.
 */
EGAT_API int egat_graph_workspace_bytes(int32_t n, size_t* bytes);
EGAT_API int egat_build_graph(const int32_t* d_pos_q, int32_t n, int32_t cutoff_q, int32_t K,
                     int32_t mode, int32_t* d_nbr_or_rowptr, int32_t* d_cnt_or_col,
                     int64_t col_capacity, int32_t* d_order, int32_t* d_overflow,
                     void* d_ws, size_t ws_bytes, void* stream);

/*
 * Step 2 — EAAS coupling ([EX] §2.1-§2.3, Proposition 4.3; [TS] §2.1, Lemma
 * 4.1, Eq. 13):
 *   y_j^{lo} = sum_{p=(li,lf,lo)} w[p][c] (x_j^{li} (x) R^{lf}(r_j))^{lo}
 * evaluated by rotating x_j into the frame whose z axis is r_j (real Wigner-D
 * matrices by the Ivanic–Ruedenberg recursion), keeping only m_i = m_o (even
 * li+lf+lo) or m_i = -m_o with sign sgn(m_o) (odd) times the Clebsch–Gordan
 * factor <li |m|; lf 0 | lo |m|> |r_j|^lf, and rotating back.
 *  d_x     [n][D][C] in s->dtype        d_pos  float32 [n][3]
 *  d_w     float32 [P][C]               d_y    [n][D][C] in s->dtype
 *                                              (bf16: round to nearest even)
 */
EGAT_API int egat_eaas_couple(const egat_shape* s, const void* d_x, const float* d_pos,
                     const float* d_w, void* d_y, void* stream);

/*
 * Step 3 — on-the-fly attention ([EX] §3.2; [TS] §2.2):
 *   s_ij^h = q_i^h . k_j^h / sqrt(dk),  alpha = softmax over j in N(i),
 *   m_i^{l}[m][c] = sum_j alpha_ij^{head(c)} h'_j^{l}[m][c]
 * streamed with an online softmax (running max and normaliser per head); each
 * neighbour's key and value rows are read once and nothing of size n*K is
 * written.  An atom without neighbours gets m_i = 0.  Neighbour entries that
 * are negative or >= n are skipped.
 *  d_q, d_k  [n][H][dk] in s->dtype      d_hp  [n][D][C] in s->dtype
 *  graph     as produced by egat_build_graph in s->graph_mode
 *            (PADDED: d_cnt may be NULL, then all K slots are scanned)
 *  d_order   optional int32 [n] traversal order (a permutation); NULL = 0..n-1
 *  d_m       float32 [n][D][C]
 */
EGAT_API int egat_otf_attention(const egat_shape* s, const void* d_q, const void* d_k,
                       const void* d_hp, const int32_t* d_nbr_or_rowptr,
                       const int32_t* d_cnt_or_col, const int32_t* d_order, float* d_m,
                       void* stream);

/*
 * Steps 3+4 fused — on-the-fly attention whose epilogue applies the target
 * coupling ^h_i = EAAS(m_i, r_i, w2) ([EX] §3.1 step 3) to the on-chip m_i
 * (m_i never reaches memory).  Arguments as egat_otf_attention, plus
 *  d_pos   float32 [n][3]      d_w2  float32 [P][C]
 *  d_out   float32 [n][D][C]   ^h
 */
EGAT_API int egat_otf_attention_coupled(const egat_shape* s, const void* d_q, const void* d_k,
                                        const void* d_hp, const int32_t* d_nbr_or_rowptr,
                                        const int32_t* d_cnt_or_col, const int32_t* d_order,
                                        const float* d_pos, const float* d_w2, float* d_out,
                                        void* stream);

/*
 * Tensor-core attention (steps 3 and 3+4 for bf16 storage, padded graphs,
 * C = 128, H = 16, dk = 16; other shapes return EGAT_ERR_UNSUPPORTED and use
 * egat_otf_attention / egat_otf_attention_coupled).  Targets are taken in
 * tiles of 16 consecutive entries of d_order (identity when NULL); one tile
 * streams the union of its targets' neighbour lists once through shared
 * memory and computes, per head, S = Q K^T and O += P V with bf16 mma.sync
 * (fp32 accumulation), the softmax restricted to each target's own
 * neighbours by a membership mask.  Same result as the per-target kernel up
 * to rounding: the softmax weights enter the P V product as bf16.
 *
 * egat_attention_plan_bytes / egat_build_attention_plan: per tile, the
 * union of the 16 targets' neighbour lists in ascending atom index, a
 * (16 x union) membership bitmask, and a target record (the 16 atom ids,
 * |r|^l and the real Wigner-D matrices of their alignment rotations for the
 * target coupling), built from the padded list (d_nbr, d_cnt — d_cnt may be
 * NULL), d_order and d_pos (float32 [n][3], required) into caller memory
 * d_plan of at least the queried size.  Per tile the builder keeps, in
 * shared memory, a bitmap over all n atoms up to n = 131,072 and beyond that
 * a hash table of the tile's candidates whose size depends on K alone; plans
 * whose shared memory would pass 200 KiB (K > 512 beyond 131,072 atoms)
 * return EGAT_ERR_UNSUPPORTED, and egat_forward then falls back to the
 * per-target kernel.  The plan depends only on the graph and the positions;
 * it is reused by every attention call on them.
 * egat_otf_attention_tiled: fused = 1 writes ^h (d_w2 required), fused = 0
 * writes m (d_w2 unused); target order and rotations come from the plan.
 * Its CTAs claim tiles at run time from a counter kept in the plan (the
 * builder zeroes it and each launch leaves it zero), so one plan serves one
 * attention launch at a time: launches that share a plan must be ordered
 * (one stream, or events); concurrent ones need plans of their own.
 */
EGAT_API int egat_attention_plan_bytes(const egat_shape* s, size_t* bytes);
EGAT_API int egat_build_attention_plan(const egat_shape* s, const int32_t* d_nbr,
                                       const int32_t* d_cnt, const int32_t* d_order,
                                       const float* d_pos, void* d_plan, size_t plan_bytes,
                                       void* stream);
/*
 * Step 2 on an attention plan — the source coupling of egat_eaas_couple for
 * every atom the plan lists, with each atom's |r|^l and Wigner-D matrices
 * read from the plan's tile records instead of being built again (the plan
 * builds them once per atom for the target coupling).  Same result as
 * egat_eaas_couple up to the rounding of the Wigner-D construction.
 *  d_plan  built by egat_build_attention_plan for the same shape and d_pos
 *  d_h, d_w1, d_hout  as egat_eaas_couple
 * Returns EGAT_ERR_UNSUPPORTED where egat_build_attention_plan would.
 */
EGAT_API int egat_eaas_couple_planned(const egat_shape* s, const void* d_h, const void* d_plan,
                                      const float* d_w1, void* d_hout, void* stream);
EGAT_API int egat_otf_attention_tiled(const egat_shape* s, const void* d_q, const void* d_k,
                                      const void* d_hp, const void* d_plan, const float* d_w2,
                                      float* d_out, int32_t fused, void* stream);

/*
 * Steps 2-4 — the fused forward pass ([EX] §3.1):
 *   h' = EAAS(h, r, w1) into workspace;  then the attention kernel streams
 *   each target's neighbours (step 3) and applies ^h_i = EAAS(m_i, r_i, w2) to
 *   the on-chip m_i before writing ^h_i.  Shapes the tensor-core path
 *   supports build the attention plan into the workspace and use
 *   egat_otf_attention_tiled; the others use the per-target kernel.
 *  d_out  float32 [n][D][C];  d_ws at least egat_forward_workspace_bytes(s).
 */
EGAT_API int egat_forward_workspace_bytes(const egat_shape* s, size_t* bytes);
EGAT_API int egat_forward(const egat_shape* s, const void* d_h, const float* d_pos, const void* d_q,
                 const void* d_k, const int32_t* d_nbr_or_rowptr, const int32_t* d_cnt_or_col,
                 const int32_t* d_order, const float* d_w1, const float* d_w2, void* d_ws,
                 size_t ws_bytes, float* d_out, void* stream);

/*
 * egat_forward_noalloc — egat_forward for callers that cannot allocate device
 * memory at call time (a plugin inside a framework that owns all device
 * allocations, a service whose memory footprint is fixed at start-up).  The
 * pages have no counterpart: this is a library convenience, not a step of the
 * method.  It takes the same arguments as egat_forward minus the workspace and
 * computes the same result; its scratch (h') lives in a library-owned device
 * array of EGAT_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library
 * holds until the process exits.  It performs no allocation.
 *  - Limit: egat_forward_workspace_bytes(s) <= EGAT_NOALLOC_SCRATCH_BYTES,
 *    i.e. h' (n * (lmax+1)^2 * C * (2 for bf16, 4 for f32) bytes, rounded up
 *    to 256) plus, for shapes on the tensor-core path, the attention plan;
 *    larger problems return EGAT_ERR_SCRATCH_LIMIT without launching.
 *  - The first call on a device, made with that device current, looks up the
 *    array's device address once (cudaGetSymbolAddress); make that first call
 *    before any stream capture.  A failed lookup returns EGAT_ERR_CUDA and is
 *    retried by the next call.  The address belongs to the device's context:
 *    after cudaDeviceReset the entry point must not be called again in that
 *    process.
 *  - All calls share the array: calls whose work overlaps on the GPU race
 *    on it and must be serialised by the caller.  Nothing in it needs
 *    clearing between calls.
 */
#define EGAT_NOALLOC_SCRATCH_BYTES (32u << 20)
EGAT_API int egat_forward_noalloc(const egat_shape* s, const void* d_h, const float* d_pos,
                                  const void* d_q, const void* d_k,
                                  const int32_t* d_nbr_or_rowptr, const int32_t* d_cnt_or_col,
                                  const int32_t* d_order, const float* d_w1, const float* d_w2,
                                  float* d_out, void* stream);

/*
 * Backward pass of steps 2-4 (the step after the forward: forces and training
 * need gradients; [EX] §3.2 keeps per-edge quantities off HBM, and so does
 * this pass: every attention weight is recomputed from q, k and one
 * log-sum-exp per target and head).  For an upstream gradient
 * G = dL/d^h (float32 [n][D][C]) of the forward egat_forward computes on the
 * padded graph (d_nbr, d_cnt; d_cnt may be NULL), writes
 *  d_dh    float32 [n][D][C]   dL/dh
 *  d_dq    float32 [n][H][dk]  dL/dq
 *  d_dk    float32 [n][H][dk]  dL/dk
 *  d_dpos  float32 [n][3]      dL/dr (forces are its negative); may be NULL, which
 *                              also skips m (on the tiled path the first pass
 *                              then streams key rows alone)
 * (positions enter through the solid harmonics of both couplings, the
 * neighbour lists held fixed; weight gradients are not computed).
 *  d_order optional int32 [n] traversal order (a permutation, as
 *          egat_build_graph returns it; NULL = 0..n-1).  It only groups atoms
 *          into tiles: results do not depend on it up to rounding, speed does.
 * Shapes of the tensor-core forward path (bf16, C = 128, H = 16, dk = 16,
 * lmax <= 3) run tiled passes: the forward kernel unfused (m and the
 * log-sum-exp), a pass over tiles of 16 targets (dq) and one over tiles of 16
 * sources and the union of the targets that list them (dk, dL/dh'; at
 * lmax 3 two sweeps of that union, one for each), with the gradient
 * products in tf32.  Other shapes gather per target and per source
 * over sorted in-lists in float32.  Either way every gradient is a sum in a
 * fixed order: deterministic, no atomics on results.  Padded graphs only (CSR
 * returns EGAT_ERR_UNSUPPORTED), n * K below 2^31; d_ws at least
 * egat_backward_workspace_bytes(s) (h', dL/dm, in-lists, per-target
 * statistics and, on the tiled path, the plans, m and dL/dh').  Errors:
 * EGAT_ERR_ARG (null or misaligned pointer), EGAT_ERR_WORKSPACE,
 * EGAT_ERR_UNSUPPORTED, EGAT_ERR_CUDA; a bounded wait that gave up is
 * reported by egat_take_device_status.
 */
EGAT_API int egat_backward_workspace_bytes(const egat_shape* s, size_t* bytes);
EGAT_API int egat_backward(const egat_shape* s, const void* d_h, const float* d_pos, const void* d_q,
                           const void* d_k, const int32_t* d_nbr, const int32_t* d_cnt,
                           const int32_t* d_order, const float* d_w1, const float* d_w2,
                           const float* d_grad_out, void* d_ws, size_t ws_bytes, float* d_dh,
                           float* d_dq, float* d_dk, float* d_dpos, void* stream);

/*
 * Invariant query/key projection ([TS] §2.2, Eq. 6: queries and keys are
 * SO(3)-invariant scalar projections of the node features; the equivariant
 * geometry travels only along the value path).  The invariant scalars of
 * atom i are its degree-0 channels h_i^(0) = d_h[i][0][0..C) (component 0 of
 * its row); each maps linearly, without bias, to every head:
 *   q[i][h][d] = sum_c h[i][0][c] wq[c][h*dk + d],   k likewise with wk,
 * so the logits q_i.k_j / sqrt(dk) are invariant.  The results feed
 * egat_otf_attention / egat_forward as d_q, d_k.
 *  d_h        [n][D][C] in s->dtype (only component 0 is read), 16-byte aligned;
 *             0 <= lmax <= 3 (D = (lmax+1)^2), K and graph_mode are ignored
 *  d_wq, d_wk float32 [C][H*dk]
 *  d_q, d_k   [n][H][dk] in s->dtype (bf16: round to nearest even)
 * bf16 storage with C = 128 and H*dk = 256 runs on tensor cores (the weights
 * as bf16 pairs hi + lo, float32 accumulation) when d_q and d_k are 16-byte
 * aligned; other shapes (C <= 1024, H*dk <= 1024) and 4-byte aligned outputs
 * accumulate in float32 on CUDA cores.  n = 0 is a no-op.
 * Errors: EGAT_ERR_ARG (null or misaligned pointer, bad dtype),
 * EGAT_ERR_UNSUPPORTED, EGAT_ERR_CUDA; a bounded wait that gave up is
 * reported by egat_take_device_status.
 */
EGAT_API int egat_qk_projection(const egat_shape* s, const void* d_h, const float* d_wq,
                                const float* d_wk, void* d_q, void* d_k, void* stream);

/*
 * Edge-centric eSCN convolution, the comparison workload (the page
 * "EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-Equivariant Graph Attention Transformers",
 * section "eSCN卷积与SO(2)线性层": rotate by D_ij from the
 * relative position, apply an SO(2) linear layer within each degree's
 * components, truncated at order M_max).  It is the edge-centric formulation
 * that the node-centric factorisation of [EX] §3.1 replaces.  For each target
 * i and each neighbour j of its padded list:
 *   r_ij = r_j - r_i, Q_ij its alignment rotation (Q_ij z = r_ij/|r_ij|, as
 *   in egat_eaas_couple; identity for r_ij = 0),
 *   x~ = D(Q_ij)^T h_j  (each degree block by its real Wigner-D matrix),
 *   per channel c, order by order (orders above mmax are zero):
 *     y~^lo_0  = sum_li W0[lo][li] x~^li_0
 *     y~^lo_+m = sum_li W1_m[lo][li] x~^li_+m - W2_m[lo][li] x~^li_-m
 *     y~^lo_-m = sum_li W2_m[lo][li] x~^li_+m + W1_m[lo][li] x~^li_-m
 *   out_i = sum_j D(Q_ij) y~.
 * Messages are summed on chip (nothing per edge is written).
 *  mmax      0 <= mmax <= lmax
 *  d_h       [n][D][C] in s->dtype, 16-byte aligned
 *  d_pos     float32 [n][3];  d_nbr / d_cnt the padded graph (d_cnt may be NULL)
 *  d_order   optional int32 [n] traversal order (NULL = 0..n-1)
 *  d_w       float32 [egat_escn_num_weights(lmax, mmax)][C]: W0 at row
 *            lo*(lmax+1) + li, then for m = 1..mmax the W1_m block followed by
 *            the W2_m block, (lmax+1-m)^2 rows each, row (lo-m)*(lmax+1-m) +
 *            (li-m) within a block
 *  d_out     float32 [n][D][C]
 * Padded graphs only (CSR returns EGAT_ERR_UNSUPPORTED).  Shapes as the
 * module header (1 <= lmax <= 3, C in {16, 32, 64, 128}).  Errors:
 * EGAT_ERR_ARG, EGAT_ERR_UNSUPPORTED, EGAT_ERR_CUDA.
 * egat_escn_num_weights returns the row count of d_w, 0 for lmax or mmax out
 * of range.
 */
EGAT_API int egat_escn_num_weights(int32_t lmax, int32_t mmax);
EGAT_API int egat_escn_conv(const egat_shape* s, int32_t mmax, const void* d_h, const float* d_pos,
                            const int32_t* d_nbr, const int32_t* d_cnt, const int32_t* d_order,
                            const float* d_w, float* d_out, void* stream);

/*
 * Row gather, the packing step of a halo exchange (a spatial domain
 * decomposition across GPUs: each rank couples its own atoms and needs the
 * h' and k rows of the neighbours it does not own; one GPU reaches about
 * 10^5 atoms, [EX] §3.2).  d_dst[r] = d_src[d_idx[r]] for r < count, rows of
 * row_bytes bytes (a positive multiple of 16), copied in 16-byte vectors; an
 * index outside [0, n_src) gives a zero row.  d_src and d_dst 16-byte
 * aligned, d_idx int32.  Asynchronous on `stream`; count = 0 is a no-op.
 * Errors: EGAT_ERR_ARG (sizes, null or misaligned pointers), EGAT_ERR_CUDA.
 */
EGAT_API int egat_gather_rows(const void* d_src, int64_t n_src, int64_t row_bytes,
                              const int32_t* d_idx, int64_t count, void* d_dst, void* stream);

/*
 * Device status.  The tensor-core attention kernel, the tile-staged source
 * coupling, the tensor-core query/key projection and the tiled backward
 * passes wait on mbarriers for their bulk copies; every such wait is bounded (about a second).  A wait that
 * gives up is counted on the device, the kernel stops waiting and finishes
 * with meaningless output instead of hanging.  The pages have no
 * counterpart: this is the library's failure report.
 *
 * egat_take_device_status: synchronises `stream`, then returns
 * EGAT_ERR_TIMEOUT if any wait gave up on the current device since the last
 * call (and clears the count), EGAT_OK otherwise, EGAT_ERR_CUDA if the
 * synchronisation or the read failed.  Call it after the work whose result
 * matters; it is not meant for a timed region.
 *
 * egat_selftest_wait_timeout: launches a one-warp kernel whose wait cannot
 * succeed (an mbarrier expecting bytes no copy delivers) and gives up after
 * `polls` polls (1 .. 1048576), so that egat_take_device_status reports
 * EGAT_ERR_TIMEOUT — a test of the failure path that faults nothing.
 * Asynchronous on `stream`; EGAT_ERR_ARG for polls out of range.
 */
EGAT_API int egat_take_device_status(void* stream);
EGAT_API int egat_selftest_wait_timeout(int32_t polls, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EGAT_H */
