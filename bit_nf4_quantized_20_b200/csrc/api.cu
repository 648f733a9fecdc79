// api.cu -- the C ABI of the library (include/qlora.h): argument validation,
// workspace layout, TMA descriptors and the launch sequence of each call.

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/qlora.h"
#include "common.cuh"
#include "kernels.h"

using namespace qlora;

namespace qlora {

// Dynamic shared memory above 48 KB needs an opt-in per kernel and per device;
// a process that drives several GPUs makes it once on each.
cudaError_t ensure_smem_optin(const void *func, int bytes) {
  struct Entry {
    const void *func;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].func == func && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (n_done < 256) done[n_done++] = Entry{func, dev, bytes};
  return cudaSuccess;
}

}  // namespace qlora

namespace {

// ---------------------------------------------------------------------------
// trace hook
// ---------------------------------------------------------------------------
struct Trace {
  qlora_trace_rec *recs = nullptr;
  int32_t cap = 0;
  int32_t *count = nullptr;
};
Trace g_trace;

enum KernelId : int32_t {
  K_QUANTIZE = 0,
  K_DEQUANTIZE = 1,
  K_LORA_U = 2,
  K_LORA_DU = 3,
  K_LORA_DB = 4,
  K_LORA_DA = 5,
  K_GEMM_FWD = 6,
  K_GEMM_BWD = 7,
  K_GEMV_FWD = 8,
  K_LORA_U_DU = 9,      // U and dU in one grid (backward)
  K_LORA_DB_DA = 10,    // dB and dA in one grid (backward)
  K_MERGE = 11,         // adapter merge for export
  K_LORA_DU_DB = 12,    // dU and dB from one read of dY (block partial sums)
  K_ADAM = 13,          // the adapters' optimizer step
  K_LORA_DU_DB_SUM = 14,  // the sums of those partials: dU planes and dB
  K_COUNT = 15,
};

const char *kKernelNames[K_COUNT] = {"quantize_nf4_dq", "dequantize_nf4", "lora_u",       "lora_du",
                                     "lora_dB",         "lora_dA",        "nf4_gemm_fwd", "nf4_gemm_bwd_dx",
                                     "nf4_gemv_fwd",    "lora_u+du",      "lora_dB+dA",   "merge_adapter",
                                     "lora_du+dB",      "adam_step",      "lora_du+dB_sum"};

struct TraceScope {
  cudaStream_t st;
  qlora_trace_rec *rec = nullptr;
  TraceScope(int32_t kernel, double flops, double bytes, cudaStream_t s) : st(s) {
    if (!g_trace.recs || !g_trace.count) return;
    const int32_t i = (*g_trace.count)++;
    if (i < g_trace.cap) {
      rec = &g_trace.recs[i];
      rec->kernel = kernel;
      rec->flops = flops;
      rec->bytes = bytes;
      if (rec->start) cudaEventRecord(static_cast<cudaEvent_t>(rec->start), st);
    }
  }
  ~TraceScope() {
    if (rec && rec->stop) cudaEventRecord(static_cast<cudaEvent_t>(rec->stop), st);
  }
};

// ---------------------------------------------------------------------------
// device properties
// ---------------------------------------------------------------------------
int num_sms_current() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Splits of the rank-r GEMMs are sized for a fixed CTA target so that the
// workspace size does not depend on the device.
constexpr int kSplitSms = 148;

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D BF16 row-major matrix [rows, cols] (row stride ld elements), box [box_rows, box_cols].
bool make_map_bf16(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows,
                   int box_cols, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status check_codebook(const float *cb) {
  for (int i = 0; i < 16; ++i)
    if (!isfinite(cb[i])) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < 15; ++i)
    if (!(cb[i] < cb[i + 1])) return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

// t_j = the smallest fp32 value >= (q_j + q_{j+1}) / 2 (midpoint formed in double):
// a normalised weight reaching t_j is at least as close to q_{j+1} as to q_j.
void snap_thresholds(const float *cb, float *thr) {
  for (int j = 0; j < 15; ++j) {
    const double mid = (static_cast<double>(cb[j]) + static_cast<double>(cb[j + 1])) * 0.5;
    float t = static_cast<float>(mid);
    if (static_cast<double>(t) < mid) t = nextafterf(t, INFINITY);
    thr[j] = t;
  }
}

// The same decisions without a division: for c1 > 0, RN32(w / c1) >= t_j holds
// exactly when w / c1 is at least the real midpoint between t_j and the next
// fp32 value below it (strictly above it when that tie rounds to the lower,
// odd neighbour).  The midpoint and the tie side per threshold, and the code of 0.
void snap_boundaries(SnapTable &tab) {
  tab.incl = 0;
  tab.snap0 = 0;
  for (int j = 0; j < 15; ++j) {
    const float t = tab.thr[j];
    const float below = nextafterf(t, -INFINITY);
    tab.mid[j] = (static_cast<double>(t) + static_cast<double>(below)) * 0.5;   // exact in double
    uint32_t bits;
    memcpy(&bits, &t, 4);
    if ((bits & 1u) == 0u) tab.incl |= 1u << j;
    if (0.0f >= t) ++tab.snap0;
  }
}

qlora_status check_weight(const qlora_nf4_weight *qw) {
  if (!qw || !qw->codes || !qw->scales || !qw->c2) return QLORA_ERR_INVALID_ARG;
  if (qw->rows <= 0 || qw->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (qw->blocksize != 64 || qw->dq_block != 256 || (qw->cols % 64) != 0) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(qw->codes)) return QLORA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(qw->c2) & 3u) != 0) return QLORA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(qw->scales) & 3u) != 0) return QLORA_ERR_MISALIGNED;
  return check_codebook(qw->codebook);
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// codebook[15 - i] == -codebook[i] bit for bit (with codebook[7] < 0 < codebook[8])
bool codebook_symmetric(const float *cb) {
  for (int i = 0; i < 8; ++i) {
    const float a = cb[i], b = -cb[15 - i];
    if (memcmp(&a, &b, sizeof(float)) != 0) return false;
  }
  return cb[7] < 0.f && cb[8] > 0.f;
}

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
// Up to this many tokens the forward runs the decode GEMV, and U = s X A^T
// runs on the mma.sync kernel (a handful of rows: latency, not bandwidth).
constexpr int64_t kGemvMaxTokens = 16;
// the decode GEMV keeps one split counter per 32-row tile in the workspace's counters
static_assert(kDecodeMaxTiles * sizeof(uint32_t) <= kWsCounterBytes, "decode tile counters");

bool decode_path(int64_t T, int64_t N) {
  (void)N;
  return T <= kGemvMaxTokens;
}

struct WsLayout {
  size_t counters = 0;
  size_t su_row = 0;                 // forward: sU hi | lo [T, 2 ceil64(r)] (rank-r operand of the GEMM / GEMV)
  size_t suT_hi = 0, suT_lo = 0;     // backward: sU^T planes [r, ceil8(T)]
  size_t du_row = 0;                 // backward: dU hi | lo [T, 2 ceil64(r)] (rank-r operand of the dX GEMM)
  size_t duT_hi = 0, duT_lo = 0;     // backward: dU^T planes [r, ceil8(T)]
  size_t bpad = 0;                   // backward: B copied to [N, ceil64(r)] when TMA cannot read it in place
  size_t partials = 0, total = 0;
};

// The split geometry of each tensor-core rank-r product (sized for kSplitSms,
// whatever the current device, so that workspace sizes are device-independent).
SkinnyTcGeom geom_u(int64_t T, int64_t K, int r) { return skinny_tc_geom(T, K, r, 1, false, kSplitSms); }
// backward: U with dU, then dB with dA, each pair in one grid
struct PairGeom {
  SkinnyTcGeom g0, g1;
  size_t part0, part1;   // partial-buffer bytes (the second starts 256-aligned after the first)
};
PairGeom pair_geom(int64_t M0, int64_t C0, bool q0, int nq0, int64_t M1, int64_t C1, bool q1, int nq1, int r) {
  PairGeom pg;
  skinny_tc_pair_geom(M0, C0, q0, nq0, M1, C1, q1, nq1, r, kSplitSms, pg.g0, pg.g1);
  pg.part0 = skinny_tc_partials_bytes(pg.g0, M0, r);
  pg.part1 = skinny_tc_partials_bytes(pg.g1, M1, r);
  return pg;
}
// U [T, r] with dU [T, r]; dB [N, r] with dA [r, K] (written as [K, r] products)
PairGeom geom_u_du(int64_t T, int64_t N, int64_t K, int r) { return pair_geom(T, K, false, 1, T, N, true, 1, r); }
PairGeom geom_db_da(int64_t T, int64_t N, int64_t K, int r) { return pair_geom(N, T, false, 2, K, T, false, 2, r); }
SkinnyTcGeom geom_da(int64_t T, int64_t K, int r) { return skinny_tc_geom(K, T, r, 2, false, kSplitSms); }
size_t pair_partials(const PairGeom &pg) {
  return static_cast<size_t>(round_up(static_cast<int64_t>(pg.part0), 256)) + pg.part1;
}

WsLayout ws_layout(int op, int64_t T, int64_t N, int64_t K, int r) {
  WsLayout L;
  size_t off = kWsHeaderBytes;
  L.counters = off;
  off += kWsCounterBytes;
  if (op == QLORA_OP_QUANTIZE) {
    L.total = off;
    return L;
  }
  const int64_t r64 = round_up(r, 64);
  const size_t row_plane = static_cast<size_t>(round_up(T * 2 * r64 * 2, 256));   // hi and lo per row
  const size_t t_plane = static_cast<size_t>(round_up(r * round_up(T, 8) * 2, 256));
  size_t part = 0;
  if (op == QLORA_OP_FWD) {
    L.su_row = off; off += row_plane;
    // the tensor-core U product (every token count when U is saved for the
    // backward, and at decode sizes when the cluster U kernel's slice does not
    // fit); at decode sizes, after it, the GEMV's split partials
    part = skinny_tc_partials_bytes(geom_u(T, K, r), T, r);
    if (decode_path(T, N)) part = std::max(part, decode_gemv_partials_bytes());
  } else {
    L.suT_hi = off; off += t_plane;
    L.suT_lo = off; off += t_plane;
    L.du_row = off; off += row_plane;
    L.duT_hi = off; off += t_plane;
    L.duT_lo = off; off += t_plane;
    L.bpad = off; off += static_cast<size_t>(round_up(N * r64 * 2, 256));
    // the paired grids of the plain backward, dA, and the fused dU/dB kernel
    // (the saved backward's two-launch dU and dB reduce in clusters: no partials)
    DuDbGeom gdd;
    const size_t p[4] = {pair_partials(geom_u_du(T, N, K, r)), pair_partials(geom_db_da(T, N, K, r)),
                         skinny_tc_partials_bytes(geom_da(T, K, r), K, r),
                         dudb_geom(T, N, r, kSplitSms, gdd) ? dudb_partials_bytes(gdd, T, N, r) : 0};
    for (size_t v : p) part = v > part ? v : part;
  }
  L.partials = off;
  off += static_cast<size_t>(round_up(static_cast<int64_t>(part), 256));
  L.total = off;
  return L;
}

// The fused GEMM's launch, prepared (tensor maps encoded, parameters filled)
// before anything of the call is enqueued.
struct GemmLaunch {
  CUtensorMap m_act, m_lact, m_act_h, m_lact_h, m_out;
  GemmParams p;
  int64_t clusters;
  int32_t kid;
  double flops, bytes;
};

qlora_status prepare_gemm(int mode, const qlora_nf4_weight *qw, const void *act, const void *lact, int64_t r64,
                          const void *lora, int r, void *out, int64_t T, uint32_t *status, GemmLaunch &g) {
  const int64_t N = qw->rows, K = qw->cols;
  const int64_t Mside = mode == 0 ? N : K;     // weight-side extent
  const int64_t Cext = mode == 0 ? K : N;      // contraction extent
  // each CTA of a pair loads 128 of a tile's 256 tokens (64 of a half tile's 128)
  if (!make_map_bf16(&g.m_act, act, T, Cext, Cext, 128, 64, true)) return QLORA_ERR_CUDA;
  if (!make_map_bf16(&g.m_lact, lact, T, 2 * r64, 2 * r64, 128, 64, true)) return QLORA_ERR_CUDA;
  if (!make_map_bf16(&g.m_act_h, act, T, Cext, Cext, 64, 64, true)) return QLORA_ERR_CUDA;
  if (!make_map_bf16(&g.m_lact_h, lact, T, 2 * r64, 2 * r64, 64, 64, true)) return QLORA_ERR_CUDA;
  // the forward stores Y by TMA from a swizzled staging tile, 128 tokens x 64 features a box
  if (mode == 0 && !make_map_bf16(&g.m_out, out, T, Mside, Mside, 128, 64, true)) return QLORA_ERR_CUDA;
  if (mode != 0) memset(&g.m_out, 0, sizeof(g.m_out));
  GemmParams &p = g.p;
  memset(&p, 0, sizeof(p));
  p.codes = qw->codes;
  p.scales = qw->scales;
  p.c2 = qw->c2;
  for (int i = 0; i < 16; ++i) p.codebook[i] = qw->codebook[i];
  p.N = N;
  p.K = K;
  p.T = T;
  p.mode = mode;
  p.lora = static_cast<const uint16_t *>(lora);
  p.r = r;
  p.m_tiles = static_cast<int>((Mside + 255) / 256);
  p.n_tiles = static_cast<int>((T + 255) / 256);
  p.k_main = static_cast<int>((Cext + 63) / 64);
  p.k_lora_plane = static_cast<int>(r64 / 64);
  p.k_lora = 2 * p.k_lora_plane;   // hi plane, then lo plane
  p.sym = codebook_symmetric(qw->codebook) ? 1 : 0;
  p.status = status;
  p.out = static_cast<uint16_t *>(out);
  p.ldo = Mside;
  g.flops = 2.0 * T * N * K + 2.0 * T * r * Mside;   // algorithmic: the lo plane's MMAs are not counted
  g.bytes = static_cast<double>(N) * K * (0.5 + 1.0 / 64) + 2.0 * T * (Cext + Mside);
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  const int sms = num_sms_current();
  g.clusters = tiles < sms / 2 ? tiles : sms / 2;
  // a last round at most half full runs its tiles as 128-token halves
  const int64_t rounds = tiles / g.clusters, rem = tiles - rounds * g.clusters;
  const bool halves = rem > 0 && rounds >= 1 && 2 * rem <= g.clusters;
  p.units_full = static_cast<int>(halves ? tiles - rem : tiles);
  p.units = static_cast<int>(halves ? tiles + rem : tiles);
  g.kid = mode == 0 ? K_GEMM_FWD : K_GEMM_BWD;
  return QLORA_OK;
}

qlora_status launch_gemm(const GemmLaunch &g, cudaStream_t st) {
  const bool fwd = g.p.mode == 0;
  const void *func = fwd ? reinterpret_cast<const void *>(nf4_gemm_fwd_2sm_kernel)
                         : reinterpret_cast<const void *>(nf4_gemm_dx_2sm_kernel);
  const int smem = fwd ? gemm_fwd_2sm_smem_bytes() : gemm_dx_2sm_smem_bytes();
  if (ensure_smem_optin(func, smem) != cudaSuccess) return QLORA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * g.clusters), 1, 1);
  cfg.blockDim = dim3(576, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  // a programmatic dependent of the rank-r kernel before it: only the loads of
  // that kernel's planes wait for it (no trace attached: with one, each launch
  // runs alone between its events)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_trace.recs == nullptr ? 2 : 1;
  TraceScope ts(g.kid, g.flops, g.bytes, st);
  const cudaError_t e =
      fwd ? cudaLaunchKernelEx(&cfg, nf4_gemm_fwd_2sm_kernel, g.m_act, g.m_lact, g.m_act_h, g.m_lact_h, g.m_out, g.p)
          : cudaLaunchKernelEx(&cfg, nf4_gemm_dx_2sm_kernel, g.m_act, g.m_lact, g.m_act_h, g.m_lact_h, g.p);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}


// 2-D byte matrix [rows, cols] (row stride ld bytes), box [box_rows, box_cols],
// with the 128-byte swizzle when box_cols == 128.
bool make_map_u8(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows,
                 int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One problem of a decode-sized launch: problem i of `a` (and of `ua`, for the
// U' kernel) from the caller's buffers; U' lives at u [T, 2 ceil64(r)].
bool fill_decode_problem(DecodeArgs &a, DecodeUArgs &ua, int i, const void *x, const qlora_nf4_weight *qw,
                         const void *A, const void *B, int r, float s, void *y, uint16_t *u, int64_t T) {
  const int64_t r64 = round_up(r, 64);
  if (!make_map_u8(&a.codes_map[i], qw->codes, qw->rows, qw->cols / 2, qw->cols / 2, 32, 128)) return false;
  DecodeProblem &p = a.prob[i];
  memset(&p, 0, sizeof(p));
  p.scales = qw->scales;
  p.c2 = qw->c2;
  for (int j = 0; j < 16; ++j) p.codebook[j] = qw->codebook[j];
  p.N = qw->rows;
  p.K = qw->cols;
  p.x = static_cast<const uint16_t *>(x);
  p.u = u;
  p.ldu = 2 * r64;
  p.B = static_cast<const uint16_t *>(B);
  p.r = r;
  p.y = static_cast<uint16_t *>(y);
  p.sym = codebook_symmetric(qw->codebook) ? 1 : 0;
  DecodeUProblem &q = ua.prob[i];
  memset(&q, 0, sizeof(q));
  q.x = static_cast<const uint16_t *>(x);
  q.A = static_cast<const uint16_t *>(A);
  q.u = u;
  q.K = qw->cols;
  q.ldu = 2 * r64;
  q.plane = r64;
  q.r = r;
  q.alpha = s;
  (void)T;
  return true;
}

double decode_bytes(const DecodeArgs &a) {
  double bytes = 0.0;
  for (int i = 0; i < a.n; ++i) {
    const DecodeProblem &p = a.prob[i];
    const double n = static_cast<double>(p.N) * p.K;
    bytes += n * (0.5 + 1.0 / 64) + 4.0 * ((n / 64 + 255) / 256) + 2.0 * a.T * (p.N + p.K) +
             2.0 * static_cast<double>(p.N) * p.r;
  }
  return bytes;
}

qlora_status run_decode_gemv(DecodeArgs &a, cudaStream_t st) {
  TraceScope ts(K_GEMV_FWD, 0.0, decode_bytes(a), st);
  // programmatic dependent launch only when no trace events sit between the kernels
  const bool pdl = g_trace.recs == nullptr;
  return launch_decode_gemv(a, num_sms_current(), st, pdl) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status run_decode_u(const DecodeUArgs &ua, cudaStream_t st) {
  double flops = 0.0, bytes = 0.0;
  for (int i = 0; i < ua.n; ++i) {
    flops += 2.0 * ua.T * ua.prob[i].K * ua.prob[i].r;
    bytes += 2.0 * ua.prob[i].r * ua.prob[i].K + 2.0 * ua.T * ua.prob[i].K;
  }
  TraceScope ts(K_LORA_U, flops, bytes, st);
  const bool pdl = g_trace.recs == nullptr;
  return launch_decode_u(ua, st, pdl) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// One tensor-core rank-r product.  P: p_col ? [C rows, M cols] : [M rows, C cols]
// (row stride ldp); Q planes: q_cj ? [C rows, R cols] : [R rows, C cols] (row
// stride ldq).  All BF16 with TMA-legal (16-byte) row strides.
struct TcProduct {
  int32_t kid;
  const void *P;
  int64_t ldp;
  bool p_col;
  const void *Q0, *Q1;
  int64_t ldq;
  bool q_cj;
  SkinnyTcGeom g;
};

// Fills the launch fields of `a` for product t (partials and counters at the
// given workspace offsets) and builds its three tensor maps {P, Q0, Q1}.
bool prepare_tc(const TcProduct &t, SkinnyTcArgs &a, uint8_t *ws, size_t part_off, size_t counter_off,
                CUtensorMap *maps) {
  a.nq = t.Q1 ? 2 : 1;
  a.p_col = t.p_col ? 1 : 0;
  a.q_cj = t.q_cj ? 1 : 0;
  a.nb = t.g.nb;
  a.stages = t.g.stages;
  a.splits = t.g.splits;
  a.c_per_split = t.g.c_per_split;
  a.partials = reinterpret_cast<float *>(ws + part_off);
  a.counters = reinterpret_cast<uint32_t *>(ws + counter_off);
  a.status = reinterpret_cast<uint32_t *>(ws);
  const bool okp = t.p_col ? make_map_bf16(&maps[0], t.P, a.C, a.M, t.ldp, 64, 64, true)
                           : make_map_bf16(&maps[0], t.P, a.M, a.C, t.ldp, 128, 64, true);
  if (!okp) return false;
  auto qmap = [&](CUtensorMap *m, const void *q) {
    return t.q_cj ? make_map_bf16(m, q, a.C, a.R, t.ldq, 64, 64, true)
                  : make_map_bf16(m, q, a.R, a.C, t.ldq, a.nb, 64, true);
  };
  if (!qmap(&maps[1], t.Q0)) return false;
  if (t.Q1) return qmap(&maps[2], t.Q1);
  maps[2] = maps[1];
  return true;
}

// A prepared tensor-core rank-r launch: one product, or two in one grid.
struct TcLaunch {
  int32_t kid;
  bool pair;
  SkinnyTcArgs a0, a1;
  CUtensorMap m0[3], m1[3];
  double flops, bytes;
};

qlora_status prepare_single_tc(const TcProduct &t, SkinnyTcArgs a, uint8_t *ws, const WsLayout &L,
                               TcLaunch &l) {
  if (!prepare_tc(t, a, ws, L.partials, L.counters, l.m0)) return QLORA_ERR_CUDA;
  a.cluster = 1;   // a single product reduces its splits inside a cluster
  l.kid = t.kid;
  l.pair = false;
  l.a0 = a;
  l.flops = 2.0 * a.M * a.C * a.R * a.nq;
  l.bytes = 2.0 * a.M * a.C;
  return QLORA_OK;
}

// Two independent products in one grid; the second's partials follow the
// first's, its counters follow the first's row tiles.
qlora_status prepare_pair_tc(int32_t kid, const TcProduct &t0, SkinnyTcArgs a0, const TcProduct &t1,
                             SkinnyTcArgs a1, const PairGeom &pg, uint8_t *ws, const WsLayout &L, TcLaunch &l) {
  const size_t part1 = L.partials + static_cast<size_t>(round_up(static_cast<int64_t>(pg.part0), 256));
  const size_t cnt1 = L.counters + static_cast<size_t>((a0.M + 127) / 128) * sizeof(uint32_t);
  if (!prepare_tc(t0, a0, ws, L.partials, L.counters, l.m0) || !prepare_tc(t1, a1, ws, part1, cnt1, l.m1))
    return QLORA_ERR_CUDA;
  l.kid = kid;
  l.pair = true;
  l.a0 = a0;
  l.a1 = a1;
  l.flops = 2.0 * (a0.M * a0.C * a0.nq + a1.M * a1.C * a1.nq) * a0.R;
  l.bytes = 2.0 * (a0.M * a0.C + a1.M * a1.C);
  return QLORA_OK;
}

qlora_status launch_tc(const TcLaunch &l, cudaStream_t st) {
  const bool pdl = g_trace.recs == nullptr;
  TraceScope ts(l.kid, l.flops, l.bytes, st);
  const cudaError_t e = l.pair ? launch_skinny_tc_pair(l.a0, l.m0, l.a1, l.m1, st, pdl)
                               : launch_skinny_tc(l.a0, l.m0[0], l.m0[1], l.m0[2], st, pdl);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

SkinnyTcArgs tc_args(int64_t M, int64_t C, int R, float alpha) {
  SkinnyTcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M;
  a.C = C;
  a.R = R;
  a.alpha = alpha;
  return a;
}

}  // namespace

extern "C" {

const char *qlora_status_string(qlora_status st) {
  switch (st) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case QLORA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_NONFINITE: return "non-finite weight";
    case QLORA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char *qlora_version(void) { return "1.0.0 sm_100a"; }

qlora_status qlora_nf4_codebook_eq2(float out[16]) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  // Phi(x) = erfc(-x / sqrt 2) / 2; its inverse by bisection to full double precision.
  auto phi = [](double x) { return 0.5 * erfc(-x / sqrt(2.0)); };
  auto inv_phi = [&](double p) {
    double lo = -12.0, hi = 12.0;
    for (int i = 0; i < 200; ++i) {
      const double mid = 0.5 * (lo + hi);
      if (phi(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
  };
  double q[16];
  for (int i = 1; i <= 16; ++i) q[i - 1] = inv_phi((i - 0.5) / 16.0);
  // normalise by the largest level; the negative half mirrors the positive one
  for (int i = 8; i < 16; ++i) {
    const float v = static_cast<float>(q[i] / q[15]);
    out[i] = v;
    out[15 - i] = -v;
  }
  return QLORA_OK;
}

qlora_status qlora_nf4_storage_bytes(int64_t rows, int64_t cols, int32_t blocksize, int32_t dq_block,
                                     size_t *codes_bytes, size_t *scales_bytes, size_t *c2_bytes) {
  if (!codes_bytes || !scales_bytes || !c2_bytes) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (blocksize != 64 || dq_block != 256 || cols % 64 != 0) return QLORA_ERR_UNSUPPORTED;
  const int64_t n = rows * cols;
  const int64_t blocks = n / 64;
  *codes_bytes = static_cast<size_t>(n / 2);
  *scales_bytes = static_cast<size_t>(blocks);
  *c2_bytes = static_cast<size_t>((blocks + 255) / 256) * 4;
  return QLORA_OK;
}

size_t qlora_workspace_bytes(int32_t op, int64_t T, int64_t N, int64_t K, int32_t r) {
  if (op == QLORA_OP_QUANTIZE) return ws_layout(op, 0, 0, 0, 1).total;
  if ((op != QLORA_OP_FWD && op != QLORA_OP_BWD) || T < 0 || N <= 0 || K <= 0 || r < 1 || r > 128) return 0;
  return ws_layout(op, T, N, K, r).total;
}

qlora_status qlora_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws || ws_bytes < kWsHeaderBytes) return QLORA_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? QLORA_OK
                                                                                              : QLORA_ERR_CUDA;
}

qlora_status qlora_get_error(void *ws, void *stream) {
  if (!ws) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return QLORA_ERR_CUDA;
  }
  if (word & DEV_TIMEOUT) return QLORA_ERR_TIMEOUT;
  if (word & DEV_NONFINITE) return QLORA_ERR_NONFINITE;
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4_ex(const void *w_bf16, int64_t rows, int64_t cols, int32_t blocksize,
                                   int32_t dq_block, const float codebook[16], uint32_t flags, qlora_nf4_weight *out,
                                   void *ws, size_t ws_bytes, void *stream) {
  if (!w_bf16 || !codebook || !out || !out->codes || !out->scales || !out->c2) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
  if ((flags & ~static_cast<uint32_t>(QLORA_QUANT_SNAP_DQ_SCALE)) != 0u) return QLORA_ERR_INVALID_ARG;
  if (blocksize != 64 || dq_block != 256 || cols % 64 != 0) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(w_bf16) || !aligned16(out->codes) || (reinterpret_cast<uintptr_t>(out->c2) & 3u))
    return QLORA_ERR_MISALIGNED;
  qlora_status cs = check_codebook(codebook);
  if (cs != QLORA_OK) return cs;
  if (!ws || ws_bytes < qlora_workspace_bytes(QLORA_OP_QUANTIZE, 0, 0, 0, 1)) return QLORA_ERR_WORKSPACE;
  out->rows = rows;
  out->cols = cols;
  out->blocksize = blocksize;
  out->dq_block = dq_block;
  SnapTable tab;
  for (int i = 0; i < 16; ++i) {
    tab.codebook[i] = codebook[i];
    out->codebook[i] = codebook[i];
  }
  snap_thresholds(codebook, tab.thr);
  snap_boundaries(tab);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nblocks = rows * cols / 64;
  const double n = static_cast<double>(rows) * cols;
  TraceScope ts(K_QUANTIZE, 0.0, n * 2.0 + n * (0.5 + 1.0 / 64) + 4.0 * ((nblocks + 255) / 256), st);
  cudaError_t e = launch_quantize(static_cast<const uint16_t *>(w_bf16), nblocks, out->codes, out->scales, out->c2,
                                  tab, (flags & QLORA_QUANT_SNAP_DQ_SCALE) != 0u, static_cast<uint32_t *>(ws), st,
                                  num_sms_current());
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_quantize_nf4(const void *w_bf16, int64_t rows, int64_t cols, int32_t blocksize,
                                int32_t dq_block, const float codebook[16], qlora_nf4_weight *out, void *ws,
                                size_t ws_bytes, void *stream) {
  return qlora_quantize_nf4_ex(w_bf16, rows, cols, blocksize, dq_block, codebook, 0u, out, ws, ws_bytes, stream);
}

qlora_status qlora_dequantize(const qlora_nf4_weight *qw, void *w_bf16_out, void *stream) {
  qlora_status s = check_weight(qw);
  if (s != QLORA_OK) return s;
  if (!w_bf16_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(w_bf16_out)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const double n = static_cast<double>(qw->rows) * qw->cols;
  TraceScope ts(K_DEQUANTIZE, 0.0, n * (0.5 + 1.0 / 64) + 4.0 * ((n / 64 + 255) / 256) + n * 2.0, st);
  cudaError_t e = launch_dequantize(qw->codes, qw->scales, qw->c2, qw->rows * qw->cols, qw->codebook,
                                    static_cast<uint16_t *>(w_bf16_out), st, num_sms_current());
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_merge_adapter(const qlora_nf4_weight *qw, const void *A, const void *B, int32_t r, float s,
                                 void *w_out, void *stream) {
  qlora_status cs = check_weight(qw);
  if (cs != QLORA_OK) return cs;
  if (!A || !B || !w_out || r < 1 || r > 128 || !isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(w_out) || (reinterpret_cast<uintptr_t>(B) & 1u)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const double n = static_cast<double>(qw->rows) * qw->cols;
  TraceScope ts(K_MERGE, 2.0 * n * r,
                n * (0.5 + 1.0 / 64) + 4.0 * ((n / 64 + 255) / 256) + 2.0 * r * (qw->rows + qw->cols) + 2.0 * n, st);
  cudaError_t e = launch_merge(qw->codes, qw->scales, qw->c2, qw->rows, qw->cols, qw->codebook,
                               static_cast<const uint16_t *>(A), static_cast<const uint16_t *>(B), r, s,
                               static_cast<uint16_t *>(w_out), st, num_sms_current());
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

static qlora_status check_linear(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                 const void *B, int32_t r, float s) {
  qlora_status st = check_weight(qw);
  if (st != QLORA_OK) return st;
  // token-sized buffers may be null (empty) when T == 0
  if ((T > 0 && !x) || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (T < 0 || r < 1 || r > 128 || !isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (qw->rows % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (T > 0x7fffffff || qw->rows > 0x7fffffff || qw->cols > 0x7fffffff) return QLORA_ERR_UNSUPPORTED;
  // decode-sized token counts keep one counter per 32 weight rows
  if (T >= 1 && decode_path(T, qw->rows) && (qw->rows + 31) / 32 > kDecodeMaxTiles) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(A) || !aligned16(B)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Every argument check of the forward that does not involve the workspace.
static qlora_status check_fwd(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A, const void *B,
                              int32_t r, float s, const void *y, const void *u_save, bool want_save) {
  qlora_status cs = check_linear(x, T, qw, A, B, r, s);
  if (cs != QLORA_OK) return cs;
  if (T > 0 && (!y || (want_save && !u_save))) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(u_save)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

static bool ws_ok(const void *ws, size_t ws_bytes, int op, int64_t T, int64_t N, int64_t K, int r) {
  return ws && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0 && ws_bytes >= qlora_workspace_bytes(op, T, N, K, r);
}

// Offsets of the two planes of a saved U (hi, then lo) for T tokens at rank r.
static size_t saved_plane_bytes(int64_t T, int r) {
  return static_cast<size_t>(round_up(static_cast<int64_t>(r) * round_up(T, 8) * 2, 256));
}

// The forward after validation (T > 0).  u_save (optional): sU^T as hi + lo
// planes [r, ceil8(T)] for the backward.
static qlora_status linear_fwd_impl(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                    const void *B, int32_t r, float s, void *y, void *u_save, void *ws,
                                    cudaStream_t st) {
  const int64_t N = qw->rows, K = qw->cols;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const WsLayout L = ws_layout(QLORA_OP_FWD, T, N, K, r);
  const int64_t r64 = round_up(r, 64);
  uint16_t *su = reinterpret_cast<uint16_t *>(w8 + L.su_row);
  const bool decode = decode_path(T, N);
  DecodeArgs da;
  DecodeUArgs ua;
  if (decode) {
    memset(&da, 0, sizeof(da));
    memset(&ua, 0, sizeof(ua));
    da.n = ua.n = 1;
    da.T = ua.T = static_cast<int>(T);
    da.part = reinterpret_cast<float *>(w8 + L.partials);
    da.counters = reinterpret_cast<uint32_t *>(w8 + L.counters);
    da.status = reinterpret_cast<uint32_t *>(ws);
    if (!fill_decode_problem(da, ua, 0, x, qw, A, B, r, s, y, su, T)) return QLORA_ERR_CUDA;
    if (!u_save && decode_u_smem_bytes(K, static_cast<int>(T)) <= kDecodeUMaxSmem) {
      // sU = s X A^T [T, hi | lo], a handful of rows: a latency-bound product on a
      // cluster kernel (one wave, partial sums in distributed shared memory)
      qlora_status rs = run_decode_u(ua, st);
      if (rs != QLORA_OK) return rs;
      da.early_start = g_trace.recs == nullptr ? 1 : 0;   // programmatic launch only without a trace
      return run_decode_gemv(da, st);
    }
  }
  // sU on the tensor cores: the row plane for the GEMM / GEMV's rank-r term
  // and, when the backward will need it, the transposed hi + lo planes
  SkinnyTcArgs au = tc_args(T, K, r, s);
  au.row_hi = su;
  au.row_lo = su + r64;
  au.ldo = 2 * r64;
  au.ocols = r64;
  if (u_save) {
    uint8_t *u8 = static_cast<uint8_t *>(u_save);
    au.t_hi = reinterpret_cast<uint16_t *>(u8);
    au.t_lo = reinterpret_cast<uint16_t *>(u8 + saved_plane_bytes(T, r));
    au.ldt = round_up(T, 8);
  }
  const TcProduct tu = {K_LORA_U, x, K, false, A, nullptr, K, false, geom_u(T, K, r)};
  TcLaunch lu;
  qlora_status rs = prepare_single_tc(tu, au, w8, L, lu);
  if (rs != QLORA_OK) return rs;
  if (decode) {
    rs = launch_tc(lu, st);
    if (rs != QLORA_OK) return rs;
    return run_decode_gemv(da, st);
  }
  GemmLaunch gl;
  rs = prepare_gemm(0, qw, x, su, r64, B, r, y, T, reinterpret_cast<uint32_t *>(ws), gl);
  if (rs != QLORA_OK) return rs;
  rs = launch_tc(lu, st);
  if (rs != QLORA_OK) return rs;
  return launch_gemm(gl, st);
}

// The backward after validation (T > 0).  u_saved (optional): the planes the
// forward saved; without them sU is recomputed from X.
static qlora_status linear_bwd_impl(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw,
                                    const void *A, const void *B, int32_t r, float s, const void *u_saved, void *dx,
                                    void *dA, void *dB, void *ws, cudaStream_t st) {
  const int64_t N = qw->rows, K = qw->cols;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const WsLayout L = ws_layout(QLORA_OP_BWD, T, N, K, r);
  const int64_t r64 = round_up(r, 64);
  const int64_t Tp = round_up(T, 8);
  auto plane = [&](size_t off) { return reinterpret_cast<uint16_t *>(w8 + off); };
  // TMA reads B in place for dU when its rows are a multiple of 16 bytes
  // (columns past r come back as zeros); otherwise B is first copied to
  // [N, ceil64(r)] rows.
  const bool pad_b = r % 8 != 0 || !aligned16(B);
  const void *bq = pad_b ? static_cast<const void *>(plane(L.bpad)) : B;
  const int64_t ldb = pad_b ? r64 : r;
  // the sU^T planes: saved by the forward, or computed below
  const uint16_t *su_hi = plane(L.suT_hi), *su_lo = plane(L.suT_lo);
  if (u_saved) {
    const uint8_t *u8 = static_cast<const uint8_t *>(u_saved);
    su_hi = reinterpret_cast<const uint16_t *>(u8);
    su_lo = reinterpret_cast<const uint16_t *>(u8 + saved_plane_bytes(T, r));
  }
  // dU = s dY B as hi | lo planes [T, 2 ceil64(r)] for the dX GEMM plus
  // transposed hi + lo planes for dA
  SkinnyTcArgs ad = tc_args(T, N, r, s);
  ad.row_hi = plane(L.du_row);
  ad.row_lo = plane(L.du_row) + r64;
  ad.ldo = 2 * r64;
  ad.ocols = r64;
  ad.t_hi = plane(L.duT_hi);
  ad.t_lo = plane(L.duT_lo);
  ad.ldt = Tp;
  // dB = dY^T (sU) [N, r] and dA = dU^T X [r, K]
  SkinnyTcArgs ab = tc_args(N, T, r, 1.0f);
  ab.row = static_cast<uint16_t *>(dB);
  SkinnyTcArgs aa = tc_args(K, T, r, 1.0f);
  aa.tr = static_cast<uint16_t *>(dA);

  TcLaunch first, mid, second, ul;
  bool have_mid = false, have_u = false;
  // r <= 64: dU and dB from one read of dY, then the sums of the blocks'
  // partials (without the saved planes, sU is computed first)
  DuDbGeom gdd;
  const bool fused = dudb_geom(T, N, r, kSplitSms, gdd);
  DuDbArgs fa;
  CUtensorMap fm_dy, fm_b, fm_su_hi, fm_su_lo;
  qlora_status rs;
  if (!u_saved && !fused) {
    // one grid: sU = s X A^T, transposed, as hi + lo planes, with dU; then
    // dB with dA in a second grid
    const PairGeom g1 = geom_u_du(T, N, K, r);
    SkinnyTcArgs au = tc_args(T, K, r, s);
    au.t_hi = plane(L.suT_hi);
    au.t_lo = plane(L.suT_lo);
    au.ldt = Tp;
    const TcProduct tu = {K_LORA_U, x, K, false, A, nullptr, K, false, g1.g0};
    const TcProduct td = {K_LORA_DU, dy, N, false, bq, nullptr, ldb, true, g1.g1};
    rs = prepare_pair_tc(K_LORA_U_DU, tu, au, td, ad, g1, w8, L, first);
    if (rs != QLORA_OK) return rs;
    const PairGeom g2 = geom_db_da(T, N, K, r);
    const TcProduct tb = {K_LORA_DB, dy, N, true, su_hi, su_lo, Tp, false, g2.g0};
    const TcProduct ta = {K_LORA_DA, x, K, true, plane(L.duT_hi), plane(L.duT_lo), Tp, false, g2.g1};
    rs = prepare_pair_tc(K_LORA_DB_DA, tb, ab, ta, aa, g2, w8, L, second);
  } else {
    if (!u_saved) {
      // sU = s X A^T as transposed hi + lo planes in the workspace, for dB
      SkinnyTcArgs au = tc_args(T, K, r, s);
      au.t_hi = plane(L.suT_hi);
      au.t_lo = plane(L.suT_lo);
      au.ldt = Tp;
      const TcProduct tu = {K_LORA_U, x, K, false, A, nullptr, K, false, geom_u(T, K, r)};
      rs = prepare_single_tc(tu, au, w8, L, ul);
      if (rs != QLORA_OK) return rs;
      have_u = true;
    }
    if (fused) {
      // dU and dB from one read of dY: block partial sums in the workspace,
      // then one launch sums them and writes dU's planes and dB
      memset(&fa, 0, sizeof(fa));
      fa.T = T;
      fa.N = N;
      fa.R = r;
      fa.tt = gdd.tt;
      fa.nn = gdd.nn;
      fa.t_ranges = gdd.t_ranges;
      fa.n_ranges = gdd.n_ranges;
      fa.rb = gdd.rb;
      fa.stages = gdd.stages;
      fa.tmem_cols = gdd.tmem_cols;
      fa.s = s;
      fa.part_u = reinterpret_cast<float *>(w8 + L.partials);
      fa.part_b = reinterpret_cast<float *>(w8 + L.partials + dudb_part_u_bytes(gdd, T, r));
      fa.du_hi = ad.row_hi;
      fa.du_lo = ad.row_lo;
      fa.ldo = ad.ldo;
      fa.ocols = ad.ocols;
      fa.duT_hi = ad.t_hi;
      fa.duT_lo = ad.t_lo;
      fa.ldt = ad.ldt;
      fa.dB = static_cast<uint16_t *>(dB);
      fa.status = reinterpret_cast<uint32_t *>(ws);
      if (!make_map_bf16(&fm_dy, dy, T, N, N, 128, 64, true) || !make_map_bf16(&fm_b, bq, N, r, ldb, 64, 64, true) ||
          !make_map_bf16(&fm_su_hi, su_hi, r, T, Tp, gdd.rb, 64, true) ||
          !make_map_bf16(&fm_su_lo, su_lo, r, T, Tp, gdd.rb, 64, true))
        return QLORA_ERR_CUDA;
    } else {
      // dB (sU comes from the forward) and dU both stream dY, as two launches
      // sharing one wave: dU is a programmatic dependent of dB that waits for
      // it only before exiting (its inputs were complete before dB started),
      // so both run at once, each reducing its splits in clusters
      SkinnyTcGeom gb, gd;
      skinny_tc_share_geom(N, T, false, 2, T, N, true, 1, r, kSplitSms, gb, gd);
      const TcProduct tb = {K_LORA_DB, dy, N, true, su_hi, su_lo, Tp, false, gb};
      const TcProduct td = {K_LORA_DU, dy, N, false, bq, nullptr, ldb, true, gd};
      rs = prepare_single_tc(tb, ab, w8, L, first);
      if (rs != QLORA_OK) return rs;
      rs = prepare_single_tc(td, ad, w8, L, mid);
      if (rs != QLORA_OK) return rs;
      mid.a0.dep_late = 1;
      have_mid = true;
    }
    // then dA
    const TcProduct ta = {K_LORA_DA, x, K, true, plane(L.duT_hi), plane(L.duT_lo), Tp, false, geom_da(T, K, r)};
    rs = prepare_single_tc(ta, aa, w8, L, second);
  }
  if (rs != QLORA_OK) return rs;
  // dX = dY W' + dU A
  GemmLaunch gl;
  rs = prepare_gemm(1, qw, dy, plane(L.du_row), r64, A, r, dx, T, reinterpret_cast<uint32_t *>(ws), gl);
  if (rs != QLORA_OK) return rs;
  // The last launch (dA, or dB with dA) needs only dU's planes and the
  // inputs, not dX: it follows the dX GEMM as a programmatic dependent that
  // waits for the GEMM only before it exits, so that it runs on the SMs the
  // GEMM's last round of tiles leaves idle.  (The GEMM lets it start after
  // the launch before the GEMM, which wrote those planes, has completed.)
  second.a0.dep_late = 1;
  second.a1.dep_late = 1;

  if (pad_b && launch_pad_cols(static_cast<const uint16_t *>(B), N, r, plane(L.bpad), static_cast<int>(r64), st,
                               num_sms_current()) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (fused) {
    const bool pdl = g_trace.recs == nullptr;
    if (have_u) {
      rs = launch_tc(ul, st);
      if (rs != QLORA_OK) return rs;
    }
    {
      TraceScope ts(K_LORA_DU_DB, 6.0 * T * N * r, 2.0 * T * N, st);
      if (launch_dudb(fa, fm_dy, fm_b, fm_su_hi, fm_su_lo, st, pdl) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    {
      const double part = 4.0 * ((r + 3) & ~3) * (static_cast<double>(fa.n_ranges) * T + static_cast<double>(fa.t_ranges) * N);
      TraceScope ts(K_LORA_DU_DB_SUM, 0.0, part + 2.0 * (2.0 * T * fa.ocols + 2.0 * r * T + static_cast<double>(N) * r), st);
      if (launch_dudb_finish(fa, st, pdl, num_sms_current()) != cudaSuccess) return QLORA_ERR_CUDA;
    }
  } else {
    rs = launch_tc(first, st);
    if (rs != QLORA_OK) return rs;
    if (have_mid) {
      rs = launch_tc(mid, st);
      if (rs != QLORA_OK) return rs;
    }
  }
  rs = launch_gemm(gl, st);
  if (rs != QLORA_OK) return rs;
  return launch_tc(second, st);
}

static qlora_status linear_bwd_entry(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw,
                                     const void *A, const void *B, int32_t r, float s, const void *u_saved,
                                     bool want_saved, void *dx, void *dA, void *dB, void *ws, size_t ws_bytes,
                                     void *stream) {
  qlora_status cs = check_linear(x, T, qw, A, B, r, s);
  if (cs != QLORA_OK) return cs;
  if ((T > 0 && (!dy || !dx || (want_saved && !u_saved))) || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(dx) || !aligned16(dA) || !aligned16(dB) || !aligned16(u_saved))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = qw->rows, K = qw->cols;
  if (!ws_ok(ws, ws_bytes, QLORA_OP_BWD, T, N, K, r)) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    // no tokens: the adapter gradients are empty sums
    if (cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  return linear_bwd_impl(dy, x, T, qw, A, B, r, s, want_saved ? u_saved : nullptr, dx, dA, dB, ws, st);
}

qlora_status qlora_linear_fwd(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A, const void *B,
                              int32_t r, float s, void *y, void *ws, size_t ws_bytes, void *stream) {
  qlora_status cs = check_fwd(x, T, qw, A, B, r, s, y, nullptr, false);
  if (cs != QLORA_OK) return cs;
  if (!ws_ok(ws, ws_bytes, QLORA_OP_FWD, T, qw->rows, qw->cols, r)) return QLORA_ERR_WORKSPACE;
  if (T == 0) return QLORA_OK;
  return linear_fwd_impl(x, T, qw, A, B, r, s, y, nullptr, ws, static_cast<cudaStream_t>(stream));
}

size_t qlora_saved_u_bytes(int64_t T, int32_t r) {
  if (T < 0 || r < 1 || r > 128) return 0;
  return 2 * saved_plane_bytes(T, r);
}

qlora_status qlora_linear_fwd_save(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                   const void *B, int32_t r, float s, void *y, void *u_save, void *ws,
                                   size_t ws_bytes, void *stream) {
  qlora_status cs = check_fwd(x, T, qw, A, B, r, s, y, u_save, true);
  if (cs != QLORA_OK) return cs;
  if (!ws_ok(ws, ws_bytes, QLORA_OP_FWD, T, qw->rows, qw->cols, r)) return QLORA_ERR_WORKSPACE;
  if (T == 0) return QLORA_OK;
  return linear_fwd_impl(x, T, qw, A, B, r, s, y, u_save, ws, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_bwd(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                              const void *B, int32_t r, float s, void *dx, void *dA, void *dB, void *ws,
                              size_t ws_bytes, void *stream) {
  return linear_bwd_entry(dy, x, T, qw, A, B, r, s, nullptr, false, dx, dA, dB, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_saved(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw,
                                    const void *A, const void *B, int32_t r, float s, const void *u_saved, void *dx,
                                    void *dA, void *dB, void *ws, size_t ws_bytes, void *stream) {
  return linear_bwd_entry(dy, x, T, qw, A, B, r, s, u_saved, true, dx, dA, dB, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// Decode-sized forward of several projections in one pair of launches
// ---------------------------------------------------------------------------
static size_t decode_batch_layout(int32_t n, const qlora_fwd_problem *probs, int64_t T, size_t *u_off,
                                  size_t *part_off) {
  size_t off = kWsHeaderBytes + kWsCounterBytes;
  for (int i = 0; i < n; ++i) {
    u_off[i] = off;
    off += static_cast<size_t>(round_up(T * 2 * round_up(probs[i].r, 64) * 2, 256));
  }
  size_t part = decode_gemv_partials_bytes();
  for (int i = 0; i < n; ++i)   // the tensor-core U fallback (a K too long for the cluster kernel)
    part = std::max(part, skinny_tc_partials_bytes(geom_u(T, probs[i].qw->cols, probs[i].r), T, probs[i].r));
  *part_off = off;
  return off + static_cast<size_t>(round_up(static_cast<int64_t>(part), 256));
}

static qlora_status check_decode_batch(int32_t n, const qlora_fwd_problem *probs, int64_t T) {
  if (n < 1 || n > kDecodeMaxProblems || !probs) return QLORA_ERR_INVALID_ARG;
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (T > kGemvMaxTokens) return QLORA_ERR_UNSUPPORTED;
  int64_t tiles = 0;
  for (int i = 0; i < n; ++i) {
    const qlora_fwd_problem &p = probs[i];
    qlora_status cs = check_fwd(p.x, T, p.qw, p.A, p.B, p.r, p.s, p.y, nullptr, false);
    if (cs != QLORA_OK) return cs;
    tiles += (p.qw->rows + 31) / 32;
  }
  if (tiles > kDecodeMaxTiles) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

size_t qlora_decode_batch_workspace_bytes(int32_t n, const qlora_fwd_problem *probs, int64_t T) {
  if (check_decode_batch(n, probs, T) != QLORA_OK) return 0;
  size_t u_off[kDecodeMaxProblems], part_off;
  return decode_batch_layout(n, probs, T, u_off, &part_off);
}

qlora_status qlora_linear_fwd_decode_batch(int32_t n, const qlora_fwd_problem *probs, int64_t T, void *ws,
                                           size_t ws_bytes, void *stream) {
  qlora_status cs = check_decode_batch(n, probs, T);
  if (cs != QLORA_OK) return cs;
  size_t u_off[kDecodeMaxProblems], part_off;
  const size_t need = decode_batch_layout(n, probs, T, u_off, &part_off);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (T == 0) return QLORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  DecodeArgs da;
  DecodeUArgs ua;
  memset(&da, 0, sizeof(da));
  memset(&ua, 0, sizeof(ua));
  da.n = n;
  da.T = ua.T = static_cast<int>(T);
  da.part = reinterpret_cast<float *>(w8 + part_off);
  da.counters = reinterpret_cast<uint32_t *>(w8 + kWsHeaderBytes);
  da.status = reinterpret_cast<uint32_t *>(ws);
  // U' of every problem: the cluster kernel for those whose K slice fits, the
  // tensor-core product for the others (prepared before anything is enqueued)
  DecodeUArgs all;
  memset(&all, 0, sizeof(all));
  TcLaunch tc[kDecodeMaxProblems];
  bool use_tc[kDecodeMaxProblems];
  for (int i = 0; i < n; ++i) {
    const qlora_fwd_problem &p = probs[i];
    uint16_t *u = reinterpret_cast<uint16_t *>(w8 + u_off[i]);
    if (!fill_decode_problem(da, all, i, p.x, p.qw, p.A, p.B, p.r, p.s, p.y, u, T)) return QLORA_ERR_CUDA;
    use_tc[i] = decode_u_smem_bytes(p.qw->cols, static_cast<int>(T)) > kDecodeUMaxSmem;
    if (use_tc[i]) {
      const int64_t r64 = round_up(p.r, 64);
      SkinnyTcArgs au = tc_args(T, p.qw->cols, p.r, p.s);
      au.row_hi = u;
      au.row_lo = u + r64;
      au.ldo = 2 * r64;
      au.ocols = r64;
      const TcProduct tu = {K_LORA_U, p.x, p.qw->cols, false, p.A, nullptr, p.qw->cols, false,
                            geom_u(T, p.qw->cols, p.r)};
      WsLayout L;
      L.counters = kWsHeaderBytes;
      L.partials = part_off;
      qlora_status rs = prepare_single_tc(tu, au, w8, L, tc[i]);
      if (rs != QLORA_OK) return rs;
    } else {
      ua.prob[ua.n++] = all.prob[i];
    }
  }
  for (int i = 0; i < n; ++i) {
    if (!use_tc[i]) continue;
    qlora_status rs = launch_tc(tc[i], st);
    if (rs != QLORA_OK) return rs;
  }
  if (ua.n > 0) {
    qlora_status rs = run_decode_u(ua, st);
    if (rs != QLORA_OK) return rs;
    da.early_start = g_trace.recs == nullptr ? 1 : 0;   // programmatic launch only without a trace
  }
  return run_decode_gemv(da, st);
}

// ---------------------------------------------------------------------------
// Forward without a caller workspace.  Its scratch (status word, split
// counters, the U' planes and the split partial sums) lives in this fixed
// device array; each GPU that loads the library reserves it until exit.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// A process-unique id of the current context (0 if the driver cannot say):
// a context created after cudaDeviceReset gets a new id.
static unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

static void *noalloc_scratch_ptr() {
  // the symbol's device address, looked up once per device and context with
  // that device current (again after the context was reset)
  static void *ptrs[64] = {nullptr};
  static unsigned long long ctx_ids[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_ctx_id();
  if (!ptrs[dev] || id == 0 || id != ctx_ids[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
    ctx_ids[dev] = id;
  }
  return ptrs[dev];
}

qlora_status qlora_linear_fwd_noalloc(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                      const void *B, int32_t r, float s, void *y, void *stream) {
  qlora_status cs = check_fwd(x, T, qw, A, B, r, s, y, nullptr, false);
  if (cs != QLORA_OK) return cs;
  const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, T, qw->rows, qw->cols, r);
  if (need == 0 || need > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_WORKSPACE;
  if (T == 0) return QLORA_OK;
  void *ws = noalloc_scratch_ptr();
  if (!ws) return QLORA_ERR_CUDA;
  // the split counters must start at zero (a call stopped by a timeout may have
  // left some set); the status word keeps what earlier calls recorded until
  // qlora_noalloc_get_error reads it
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<uint8_t *>(ws) + kWsHeaderBytes, 0, kWsCounterBytes, st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return linear_fwd_impl(x, T, qw, A, B, r, s, y, nullptr, ws, st);
}

qlora_status qlora_noalloc_get_error(void *stream) {
  void *ws = noalloc_scratch_ptr();
  if (!ws) return QLORA_ERR_CUDA;
  return qlora_get_error(ws, stream);
}

// ---------------------------------------------------------------------------
// Failure-detection self-test: one thread waits, with the same bounded wait
// every pipeline of the library uses, on an mbarrier that no thread arrives on.
// The wait gives up after limit_ns and records DEV_TIMEOUT in the status word.
// ---------------------------------------------------------------------------
static __global__ void wait_selftest_kernel(uint32_t *status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // parity 0 of a fresh barrier completes only after one arrival, which never comes
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, status, limit_ns);
  __syncthreads();
}

qlora_status qlora_wait_selftest(void *ws, size_t ws_bytes, uint32_t limit_us, void *stream) {
  if (ws && (ws_bytes < kWsHeaderBytes || (reinterpret_cast<uintptr_t>(ws) & 255u))) return QLORA_ERR_WORKSPACE;
  if (limit_us == 0 || limit_us > 2000000u) return QLORA_ERR_INVALID_ARG;
  if (!ws) ws = noalloc_scratch_ptr();   // the allocation-free forward's status word
  if (!ws) return QLORA_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t *>(ws),
                                                                        1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// The adapters' optimizer step and its unified-memory ("paged") state
// ---------------------------------------------------------------------------
qlora_status qlora_adam_step(float *param, float *m, float *v, const void *grad_bf16, void *param_bf16, int64_t n,
                             const qlora_adam_hparams *h, void *stream) {
  if (!h || n < 0) return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!param || !m || !v || !grad_bf16) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(param) || !aligned16(m) || !aligned16(v) || !aligned16(grad_bf16) || !aligned16(param_bf16))
    return QLORA_ERR_MISALIGNED;
  if (h->step < 1 || !isfinite(h->lr) || !isfinite(h->eps) || !isfinite(h->weight_decay) || !(h->eps > 0.f) ||
      !(h->beta1 >= 0.f && h->beta1 < 1.f) || !(h->beta2 >= 0.f && h->beta2 < 1.f))
    return QLORA_ERR_INVALID_ARG;
  AdamArgs a;
  a.lr = h->lr;
  a.beta1 = h->beta1;
  a.beta2 = h->beta2;
  a.one_minus_beta1 = static_cast<float>(1.0 - static_cast<double>(h->beta1));
  a.one_minus_beta2 = static_cast<float>(1.0 - static_cast<double>(h->beta2));
  a.eps = h->eps;
  a.decay = static_cast<float>(1.0 - static_cast<double>(h->lr) * h->weight_decay);
  a.bc1 = static_cast<float>(1.0 - pow(static_cast<double>(h->beta1), h->step));
  a.bc2 = static_cast<float>(1.0 - pow(static_cast<double>(h->beta2), h->step));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TraceScope ts(K_ADAM, 0.0, 28.0 * n - (param_bf16 ? 0.0 : 2.0 * n), st);
  return launch_adam(param, m, v, static_cast<const uint16_t *>(grad_bf16), static_cast<uint16_t *>(param_bf16), n,
                     a, st, num_sms_current()) == cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_alloc(size_t bytes, void **ptr) {
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  *ptr = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  void *p = nullptr;
  if (cudaMallocManaged(&p, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  // live on this GPU while there is room; the driver pages out under pressure
  (void)cudaMemAdvise(p, bytes, cudaMemAdviseSetPreferredLocation, dev);
  (void)cudaGetLastError();
  *ptr = p;
  return QLORA_OK;
}

qlora_status qlora_paged_free(void *ptr) {
  if (!ptr) return QLORA_OK;
  return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_prefetch(void *ptr, size_t bytes, int32_t to_host, void *stream) {
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  if (!to_host && cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  return cudaMemPrefetchAsync(ptr, bytes, to_host ? cudaCpuDeviceId : dev, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

qlora_status qlora_trace_attach(qlora_trace_rec *recs, int32_t capacity, int32_t *count) {
  if (recs && (!count || capacity < 0)) return QLORA_ERR_INVALID_ARG;
  g_trace.recs = recs;
  g_trace.cap = recs ? capacity : 0;
  g_trace.count = recs ? count : nullptr;
  return QLORA_OK;
}

const char *qlora_kernel_name(int32_t kernel) {
  if (kernel < 0 || kernel >= K_COUNT) return "unknown";
  return kKernelNames[kernel];
}

}  // extern "C"
