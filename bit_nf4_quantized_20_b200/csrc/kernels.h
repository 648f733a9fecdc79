// kernels.h -- parameter blocks and launch helpers shared between the C-ABI
// layer (api.cu) and the kernels.  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

// Codebook and its snapping thresholds, passed by value to the quantizer.
struct SnapTable {
  float codebook[16];
  float thr[15];   // t_j = smallest fp32 >= (q_j + q_{j+1}) / 2
  // RN32(x) >= t_j  <=>  x >= mid_j (incl bit j set) or x > mid_j (clear), with
  // mid_j the real midpoint between t_j and the fp32 value below it (ties to even)
  double mid[15];
  uint32_t incl;
  uint32_t snap0;  // the code of w_hat = 0 (all-zero blocks)
};

// ---------------------------------------------------------------------------
// quantize / dequantize (quant.cu)
// ---------------------------------------------------------------------------
// out[N, K] = BF16(W' + s B A) (quant.cu)
cudaError_t launch_merge(const uint8_t *codes, const uint8_t *scales, const float *c2, int64_t N, int64_t K,
                         const float (&codebook)[16], const uint16_t *A, const uint16_t *B, int r, float s,
                         uint16_t *out, cudaStream_t st, int num_sms);
// snap_dq: codes snapped against the double-quantized scale s_b instead of c1
cudaError_t launch_quantize(const uint16_t *w, int64_t n_blocks, uint8_t *codes, uint8_t *scales, float *c2,
                            const SnapTable &tab, bool snap_dq, uint32_t *status, cudaStream_t st, int num_sms);
cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales, const float *c2, int64_t n_weights,
                              const float (&codebook)[16], uint16_t *out, cudaStream_t st, int num_sms);

// Opt `func` in to `bytes` of dynamic shared memory on the current device, once
// per (function, device); thread-safe (api.cu).
cudaError_t ensure_smem_optin(const void *func, int bytes);

// ---------------------------------------------------------------------------
// the adapters' optimizer step (optim.cu): Adam with decoupled weight decay
// ---------------------------------------------------------------------------
struct AdamArgs {
  float lr, beta1, beta2, one_minus_beta1, one_minus_beta2, eps;
  float decay;      // 1 - lr * weight_decay
  float bc1, bc2;   // 1 - beta1^step, 1 - beta2^step
};
cudaError_t launch_adam(float *param, float *m, float *v, const uint16_t *grad, uint16_t *out_bf16, int64_t n,
                        const AdamArgs &a, cudaStream_t st, int num_sms);

// ---------------------------------------------------------------------------
// fused NF4 GEMMs on CTA pairs (gemm_fwd_2sm.cu, gemm_dx_2sm.cu)
// ---------------------------------------------------------------------------
struct GemmParams {
  const uint8_t *codes;
  const uint8_t *scales;
  const float *c2;
  float codebook[16];
  int64_t N, K;            // quantized weight is N x K
  int64_t T;               // tokens
  int mode;                // 0: forward (M side = N rows), 1: backward dX (M side = K columns)
  const uint16_t *lora;    // forward: B[N, r]; backward: A[r, K]
  int r;
  int m_tiles, n_tiles;    // weight-side tiles of 256 (one CTA pair), token tiles of 256
  // Work units, in order: tiles 0 .. units_full - 1 whole (tile t: weight tile
  // t % m_tiles, token tile t / m_tiles), then each remaining tile as two
  // 128-token halves (units - units_full of them), so that a last round that
  // would leave most CTA pairs idle takes half as long.
  int units, units_full;
  int k_main, k_lora;      // 64-wide contraction stages: weight part, rank-r part (hi then lo plane)
  int k_lora_plane;        // rank-r stages per plane (k_lora = 2 k_lora_plane)
  int sym;                 // codebook[15 - i] == -codebook[i] exactly (8-entry lookup)
  uint32_t *status;
  uint16_t *out;           // Y [T, N] (stored by TMA through tmap_out) or dX [T, K] (from registers)
  int64_t ldo;             // its row stride (N or K)
};
// Launched as clusters of 2 CTAs, one CTA per SM, persistent over the work
// units.  Token operand maps: act = X or dY [T, C], lact = the rank-r planes
// [T, 2 ceil64(r)]; boxes of 64 columns by 128 rows (whole tiles: each CTA
// loads half of 256 tokens) or by 64 rows (the "_h" maps: half tiles),
// 128-byte swizzle.
// The forward (mode 0), A from tensor memory; tmap_out: Y [T, N], box [128
// tokens][64 features], 128-byte swizzle (gemm_fwd_2sm.cu).
int gemm_fwd_2sm_smem_bytes();
__global__ void nf4_gemm_fwd_2sm_kernel(const __grid_constant__ CUtensorMap tmap_act,
                                        const __grid_constant__ CUtensorMap tmap_lact,
                                        const __grid_constant__ CUtensorMap tmap_act_h,
                                        const __grid_constant__ CUtensorMap tmap_lact_h,
                                        const __grid_constant__ CUtensorMap tmap_out, const GemmParams p);
// The backward dX (mode 1), A = W'^T from shared memory (gemm_dx_2sm.cu).
int gemm_dx_2sm_smem_bytes();
__global__ void nf4_gemm_dx_2sm_kernel(const __grid_constant__ CUtensorMap tmap_act,
                                       const __grid_constant__ CUtensorMap tmap_lact,
                                       const __grid_constant__ CUtensorMap tmap_act_h,
                                       const __grid_constant__ CUtensorMap tmap_lact_h, const GemmParams p);

// ---------------------------------------------------------------------------
// decode-sized forward of one or several projections (decode.cu)
// ---------------------------------------------------------------------------
constexpr int kDecodeMaxProblems = 8;
constexpr int kDecodeWarps = 6;
constexpr int kDecodeMaxCtas = 512;
constexpr int64_t kDecodeMaxTiles = 16384;       // 32-row tiles over all problems (workspace counters)
constexpr int kDecodeUMaxSmem = 200 * 1024;

struct DecodeProblem {
  const uint8_t *scales;
  const float *c2;
  float codebook[16];
  int64_t N, K;
  int64_t kb;            // K / 64 blocks per row                        (filled by the launcher)
  int kus;               // 256-code units per row                        (filled by the launcher)
  int64_t tiles;         // 32-row tiles                                  (filled by the launcher)
  int64_t unit0, tile0;  // first global unit and tile of this problem    (filled by the launcher)
  const uint16_t *x;     // [T, K]
  const uint16_t *u;     // U' = s X A^T as hi | lo BF16 planes per row [T, ldu]
  int64_t ldu;
  const uint16_t *B;     // [N, r]
  int r;
  uint16_t *y;           // [T, N]
  int sym;               // codebook[15 - i] == -codebook[i] exactly (8-entry lookup)
};
struct __align__(64) DecodeArgs {
  CUtensorMap codes_map[kDecodeMaxProblems];   // codes as bytes [N][K / 2], box [32 rows][128 B], 128-byte swizzle
  DecodeProblem prob[kDecodeMaxProblems];
  int n, T;
  int early_start;       // the preceding kernel is decode_u_kernel: stream before the dependency wait
  int64_t units;         // (filled by the launcher)
  float *part;           // [kDecodeMaxCtas][2][16][32] fp32: sums of tiles that straddle CTAs
  uint32_t *counters;    // one per tile over all problems (zero between calls)
  uint32_t *status;
};
size_t decode_gemv_partials_bytes();
cudaError_t launch_decode_gemv(DecodeArgs &a, int num_sms, cudaStream_t st, bool pdl);

struct DecodeUProblem {
  const uint16_t *x;     // [T, K]
  const uint16_t *A;     // [r, K]
  uint16_t *u;           // [T, ldu]: hi plane in columns 0 .. plane - 1, lo plane from column plane
  int64_t K, ldu, plane; // plane a multiple of 16, >= r
  int r;
  float alpha;
  int kc, cluster0;      // (filled by the launcher)
};
struct DecodeUArgs {
  DecodeUProblem prob[kDecodeMaxProblems];
  int n, T;
  int red_off;           // (filled by the launcher)
};
// Dynamic shared memory of decode_u_kernel for the longest K of a launch; the
// kernel runs when it is <= kDecodeUMaxSmem.
int decode_u_smem_bytes(int64_t K_max, int T);
cudaError_t launch_decode_u(const DecodeUArgs &a, cudaStream_t st, bool pdl);

// ---------------------------------------------------------------------------
// the rank-r LoRA products (skinny_tc.cu):
//   C[M, R] = alpha * sum_c P(m, c) * Q(c, j),  Q = Q0 (+ Q1)
// P and Q arrive by TMA, the accumulator (128 rows x NB columns, FP32) lives in
// tensor memory.
// ---------------------------------------------------------------------------
struct SkinnyTcGeom {
  int nb;               // MMA N: R rounded up to 16, 32, 64 or 128 (64 or 128 for MN-major Q)
  int stages;           // TMA pipeline depth
  int smem;             // dynamic shared memory bytes
  int splits;           // contraction splits (CTAs per 128-row tile)
  int64_t c_per_split;  // multiple of 64
};
// nq: Q planes (1, or 2 for hi + lo); q_cj: Q stored [c][j] (MN-major) else [j][c].
// At most kSkinnyMaxClusterSplits splits, so that a launch of one product can
// reduce its splits inside a thread-block cluster.
constexpr int kSkinnyMaxClusterSplits = 8;
SkinnyTcGeom skinny_tc_geom(int64_t M, int64_t C, int R, int nq, bool q_cj, int num_sms);
// Two products launched one after the other to run side by side in one wave:
// each with its own tile width and pipeline depth, the CTA slots shared in
// proportion to their bytes, at most kSkinnyMaxClusterSplits splits each.
void skinny_tc_share_geom(int64_t M0, int64_t C0, bool q_cj0, int nq0, int64_t M1, int64_t C1, bool q_cj1, int nq1,
                          int R, int num_sms, SkinnyTcGeom &g0, SkinnyTcGeom &g1);
size_t skinny_tc_partials_bytes(const SkinnyTcGeom &g, int64_t M, int R);

struct SkinnyTcArgs {
  int64_t M, C;          // rows of the result, contraction length
  int R;                 // result columns (<= 128)
  int nq;                // Q planes summed into one accumulator
  int p_col;             // P stored [c][m] (MN-major A) else [m][c] (K-major A)
  int q_cj;              // Q stored [c][j] (MN-major B) else [j][c] (K-major B)
  int nb, stages, splits;
  int64_t c_per_split;
  float alpha;
  // outputs (nullptr = not written); v = alpha * C[m, j]
  uint16_t *row_hi;      // [M, ldo] bf16(v), columns R..ocols-1 zero
  uint16_t *row_lo;      // [M, ldo] bf16(v - bf16(v)), columns R..ocols-1 zero (optional)
  int64_t ldo, ocols;    // row stride; columns written per row (ocols <= ldo)
  uint16_t *t_hi;        // [R, ldt] bf16(v) transposed
  uint16_t *t_lo;        // [R, ldt] bf16(v - bf16(v)) transposed
  int64_t ldt;
  uint16_t *row;         // [M, R] bf16(v)
  uint16_t *tr;          // [R, M] bf16(v)
  float *partials;       // [splits][M][(R + 3) & ~3] when splits > 1
  uint32_t *counters;    // one per 128-row tile (zero on entry, zero on exit)
  uint32_t *status;
  int cluster;           // single-product launches with splits <= 8: the splits of a row tile are
                         // one cluster and reduce through distributed shared memory (no partials,
                         // no counters)
  int dep_late;          // every input was complete when the preceding kernel let this one
                         // start: wait for that kernel only before exiting (same in both
                         // products of a pair launch)
};
cudaError_t launch_skinny_tc(const SkinnyTcArgs &a, const CUtensorMap &tm_p, const CUtensorMap &tm_q0,
                             const CUtensorMap &tm_q1, cudaStream_t st, bool pdl);
// Two independent products sharing one wave -- in one grid (the pair launch),
// or as two launches that run side by side -- with one tile width (the larger
// of the two), the CTA slots of the wave shared in proportion to their bytes.
// Both have R columns; each has its own Q plane count (nq0, nq1), pipeline
// depth, partials and counters.  max_splits > 0 caps each product's splits.
void skinny_tc_pair_geom(int64_t M0, int64_t C0, bool q_cj0, int nq0, int64_t M1, int64_t C1, bool q_cj1, int nq1,
                         int R, int num_sms, SkinnyTcGeom &g0, SkinnyTcGeom &g1, int max_splits = 0);
// maps: {P, Q0, Q1} for each product
cudaError_t launch_skinny_tc_pair(const SkinnyTcArgs &a0, const CUtensorMap *maps0, const SkinnyTcArgs &a1,
                                  const CUtensorMap *maps1, cudaStream_t st, bool pdl);
cudaError_t launch_pad_cols(const uint16_t *src, int64_t rows, int cols, uint16_t *dst, int ldd, cudaStream_t st,
                            int num_sms);

// ---------------------------------------------------------------------------
// dU = s dY B and dB = dY^T (sU) from one read of dY (dudb.cu), for r <= 64:
// each CTA streams a block of dY (tt 128-token tiles x nn 128-feature chunks)
// once, both accumulators in tensor memory; the blocks' FP32 partial sums go
// to the workspace and a second launch sums them and writes the outputs.
// ---------------------------------------------------------------------------
constexpr int kDudbMaxRank = 64;
constexpr int kDudbMaxStages = 8;
constexpr int kDudbMaxChunks = 32;
struct DuDbGeom {
  int tt, nn;                  // 128-token tiles, 128-feature chunks per CTA
  int t_ranges, n_ranges;      // the grid: t_ranges x n_ranges CTAs
  int rb;                      // r rounded up to 16, 32 or 64: the hi and lo sU planes stacked
                               // make a 2 rb-column dB accumulator
  int stages;                  // dY tiles in flight (32 KiB each)
  int smem;                    // dynamic shared memory bytes
  int tmem_cols;               // tensor-memory columns allocated (a power of two)
};
// false: the shape is not covered (r > kDudbMaxRank, or no geometry fits).
bool dudb_geom(int64_t T, int64_t N, int r, int num_sms, DuDbGeom &g);
// the two partial-sum buffers: dU [n_ranges][T][(r + 3) & ~3], then (256-aligned)
// dB [t_ranges][N][(r + 3) & ~3], FP32
size_t dudb_part_u_bytes(const DuDbGeom &g, int64_t T, int r);
size_t dudb_partials_bytes(const DuDbGeom &g, int64_t T, int64_t N, int r);

struct DuDbArgs {
  int64_t T, N;
  int R;
  int tt, nn, t_ranges, n_ranges, rb, stages, tmem_cols;
  float s;                     // dU = s dY B (dB takes sU, already scaled)
  float *part_u;               // [n_ranges][T][(R + 3) & ~3]
  float *part_b;               // [t_ranges][N][(R + 3) & ~3]
  // outputs of the second launch; v = s dU-sum
  uint16_t *du_hi, *du_lo;     // [T, ldo] bf16(v) and bf16(v - bf16(v)), columns R..ocols-1 zero
  int64_t ldo, ocols;          // ocols a multiple of 4
  uint16_t *duT_hi, *duT_lo;   // [R, ldt] the same, transposed
  int64_t ldt;
  uint16_t *dB;                // [N, R]
  uint32_t *status;
};
// maps: dY [T rows, N cols] box 128 x 64; B as [N rows, R cols] box 64 x 64
// (columns past R read as zeros); the sU^T planes [R rows, T cols] box rb x 64.
cudaError_t launch_dudb(const DuDbArgs &a, const CUtensorMap &tm_dy, const CUtensorMap &tm_b,
                        const CUtensorMap &tm_su_hi, const CUtensorMap &tm_su_lo, cudaStream_t st, bool pdl);
cudaError_t launch_dudb_finish(const DuDbArgs &a, cudaStream_t st, bool pdl, int num_sms);

}  // namespace qlora
