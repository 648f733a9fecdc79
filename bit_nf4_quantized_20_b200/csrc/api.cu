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
  K_COUNT = 12,
};

const char *kKernelNames[K_COUNT] = {"quantize_nf4_dq", "dequantize_nf4", "lora_u",       "lora_du",
                                     "lora_dB",         "lora_dA",        "nf4_gemm_fwd", "nf4_gemm_bwd_dx",
                                     "nf4_gemv_fwd",    "lora_u+du",      "lora_dB+dA",   "merge_adapter"};

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

// A second stream (and its fork / join events) per host thread and device: the
// backward runs its adapter-gradient products there, beside the dX GEMM, whose
// last partial round of tiles leaves SMs idle.  Created on first use, kept
// until exit; nullptr if the device refuses (the caller then stays on one stream).
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool tried = false;
};

SideStream *side_stream() {
  thread_local SideStream cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream &ss = cache[dev];
  if (!ss.tried) {
    ss.tried = true;
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      ss.s = nullptr;
      (void)cudaGetLastError();
    }
  }
  return ss.s ? &ss : nullptr;
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
// the split counters of the decode GEMV are the workspace's tile counters
constexpr int kGemvMaxCounterTiles = static_cast<int>(kWsCounterBytes / sizeof(uint32_t));

bool decode_path(int64_t T, int64_t N) {
  (void)N;
  return T <= kGemvMaxTokens;
}

struct WsLayout {
  size_t counters = 0;
  size_t su_row = 0;                 // forward: sU [T, ceil64(r)] (rank-r operand of the GEMM / GEMV)
  size_t suT_hi = 0, suT_lo = 0;     // backward: sU^T planes [r, ceil8(T)]
  size_t du_row = 0;                 // backward: dU hi [T, ceil64(r)] (rank-r operand of the dX GEMM)
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
PairGeom pair_geom(int64_t M0, int64_t C0, bool q0, int64_t M1, int64_t C1, bool q1, int r, int nq) {
  PairGeom pg;
  skinny_tc_pair_geom(M0, C0, q0, M1, C1, q1, r, nq, kSplitSms, pg.g0, pg.g1);
  pg.part0 = skinny_tc_partials_bytes(pg.g0, M0, r);
  pg.part1 = skinny_tc_partials_bytes(pg.g1, M1, r);
  return pg;
}
PairGeom geom_u_du(int64_t T, int64_t N, int64_t K, int r) { return pair_geom(T, K, false, T, N, true, r, 1); }
PairGeom geom_db_da(int64_t T, int64_t N, int64_t K, int r) { return pair_geom(N, T, false, K, T, false, r, 2); }
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
  const size_t row_plane = static_cast<size_t>(round_up(T * r64 * 2, 256));
  const size_t t_plane = static_cast<size_t>(round_up(r * round_up(T, 8) * 2, 256));
  size_t part = 0;
  if (op == QLORA_OP_FWD) {
    L.su_row = off; off += row_plane;
    if (decode_path(T, N)) {
      // the U' fallback's partials, then (after it has finished) the GEMV's split partials
      part = std::max(skinny_partials_bytes(T, K, r, kSplitSms),
                      gemv_persist_partials_bytes(N, K, kGemvMaxCounterTiles));
    } else {
      part = skinny_tc_partials_bytes(geom_u(T, K, r), T, r);
    }
  } else {
    L.suT_hi = off; off += t_plane;
    L.suT_lo = off; off += t_plane;
    L.du_row = off; off += row_plane;
    L.duT_hi = off; off += t_plane;
    L.duT_lo = off; off += t_plane;
    L.bpad = off; off += static_cast<size_t>(round_up(N * r64 * 2, 256));
    const size_t p[2] = {pair_partials(geom_u_du(T, N, K, r)), pair_partials(geom_db_da(T, N, K, r))};
    for (size_t v : p) part = v > part ? v : part;
  }
  L.partials = off;
  off += static_cast<size_t>(round_up(static_cast<int64_t>(part), 256));
  L.total = off;
  return L;
}

// Parameters of the mma.sync rank-r kernel (decode-sized U only).
SkinnyParams skinny_base(int64_t M, int64_t C, int R, uint8_t *ws, const WsLayout &L) {
  SkinnyParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.C = C;
  p.R = R;
  p.splits = skinny_splits(M, C, kSplitSms);
  int64_t per = (C + p.splits - 1) / p.splits;
  p.c_per_split = round_up(per, 64);
  p.partials = reinterpret_cast<float *>(ws + L.partials);
  p.counters = reinterpret_cast<uint32_t *>(ws + L.counters);
  p.status = reinterpret_cast<uint32_t *>(ws);
  return p;
}

// The one-CTA GEMM kernel is kept for comparison measurements; setting
// QLORA_GEMM_ONE_CTA=1 in the environment selects it.
bool use_one_cta_gemm() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("QLORA_GEMM_ONE_CTA");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

qlora_status run_gemm(int mode, const qlora_nf4_weight *qw, const void *act, const void *lact, int64_t r64,
                      const void *lora, int r, void *out, int64_t T, uint32_t *status, cudaStream_t st) {
  const int64_t N = qw->rows, K = qw->cols;
  const int64_t Mside = mode == 0 ? N : K;     // weight-side extent
  const int64_t Cext = mode == 0 ? K : N;      // contraction extent
  // the CTA-pair kernel (default) loads 128 tokens per CTA; the one-CTA kernel 256
  const bool pair = !use_one_cta_gemm();
  const int act_rows = pair ? 128 : 256;
  CUtensorMap m_act, m_lact, m_out;
  if (!make_map_bf16(&m_act, act, T, Cext, Cext, act_rows, 64, true)) return QLORA_ERR_CUDA;
  if (!make_map_bf16(&m_lact, lact, T, r64, r64, act_rows, 64, true)) return QLORA_ERR_CUDA;
  if (!make_map_bf16(&m_out, out, T, Mside, Mside, 32, 128, false)) return QLORA_ERR_CUDA;
  GemmParams p;
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
  p.m_tiles = static_cast<int>((Mside + (pair ? 255 : 127)) / (pair ? 256 : 128));
  p.n_tiles = static_cast<int>((T + 255) / 256);
  p.k_main = static_cast<int>((Cext + 63) / 64);
  p.k_lora = static_cast<int>(r64 / 64);
  p.sym = codebook_symmetric(qw->codebook) ? 1 : 0;
  p.status = status;
  p.out = static_cast<uint16_t *>(out);
  p.ldo = Mside;
  const double flops = 2.0 * T * N * K + 2.0 * T * r * Mside;
  const double bytes = static_cast<double>(N) * K * (0.5 + 1.0 / 64) + 2.0 * T * (Cext + Mside);
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  const int sms = num_sms_current();
  if (pair) {
    static bool attr2 = false;
    if (!attr2) {
      if (cudaFuncSetAttribute(nf4_gemm_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               gemm_2sm_smem_bytes()) != cudaSuccess)
        return QLORA_ERR_CUDA;
      attr2 = true;
    }
    const int64_t clusters = tiles < sms / 2 ? tiles : sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    cfg.blockDim = dim3(576, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(gemm_2sm_smem_bytes());
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceScope ts(mode == 0 ? K_GEMM_FWD : K_GEMM_BWD, flops, bytes, st);
    return cudaLaunchKernelEx(&cfg, nf4_gemm_2sm_kernel, m_act, m_lact, m_out, p) == cudaSuccess ? QLORA_OK
                                                                                                  : QLORA_ERR_CUDA;
  }
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(nf4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes()) !=
        cudaSuccess)
      return QLORA_ERR_CUDA;
    attr_set = true;
  }
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  TraceScope ts(mode == 0 ? K_GEMM_FWD : K_GEMM_BWD, flops, bytes, st);
  nf4_gemm_kernel<<<grid, 320, gemm_smem_bytes(), st>>>(m_act, m_lact, m_out, p);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}


// The decode forward; u holds U' = BF16(s X A^T) [T, ldu].
qlora_status run_gemv(const qlora_nf4_weight *qw, const void *x, int64_t T, const uint16_t *u, int64_t ldu,
                      const void *B, int r, void *y, uint8_t *ws, const WsLayout &L, cudaStream_t st) {
  GemvParams p;
  memset(&p, 0, sizeof(p));
  p.codes = qw->codes;
  p.scales = qw->scales;
  p.c2 = qw->c2;
  for (int i = 0; i < 16; ++i) p.codebook[i] = qw->codebook[i];
  p.N = qw->rows;
  p.K = qw->cols;
  p.T = static_cast<int>(T);
  p.x = static_cast<const uint16_t *>(x);
  p.u = u;
  p.ldu = ldu;
  p.B = static_cast<const uint16_t *>(B);
  p.r = r;
  p.y = static_cast<uint16_t *>(y);
  p.sym = codebook_symmetric(qw->codebook) ? 1 : 0;
  p.ctas = gemv_persist_ctas(p.N, p.K, num_sms_current(), kGemvMaxCounterTiles);
  p.part = reinterpret_cast<float *>(ws + L.partials);
  p.counters = reinterpret_cast<uint32_t *>(ws + L.counters);
  const double n = static_cast<double>(p.N) * p.K;
  const double bytes = n * (0.5 + 1.0 / 64) + 4.0 * ((n / 64 + 255) / 256) + 2.0 * T * (p.N + p.K) +
                       2.0 * static_cast<double>(p.N) * r;
  TraceScope ts(K_GEMV_FWD, 0.0, bytes, st);
  // programmatic dependent launch only when no trace events sit between the kernels
  const bool pdl = g_trace.recs == nullptr;
  return launch_gemv(p, num_sms_current(), st, pdl) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
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

qlora_status run_skinny_tc(const TcProduct &t, SkinnyTcArgs a, uint8_t *ws, const WsLayout &L, cudaStream_t st) {
  CUtensorMap maps[3];
  if (!prepare_tc(t, a, ws, L.partials, L.counters, maps)) return QLORA_ERR_CUDA;
  const double flops = 2.0 * a.M * a.C * a.R * a.nq;
  const double bytes = 2.0 * a.M * a.C;
  const bool pdl = g_trace.recs == nullptr;
  TraceScope ts(t.kid, flops, bytes, st);
  return launch_skinny_tc(a, maps[0], maps[1], maps[2], st, pdl) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Two independent products in one grid; the second's partials follow the
// first's, its counters follow the first's row tiles.
qlora_status run_skinny_tc_pair(int32_t kid, const TcProduct &t0, SkinnyTcArgs a0, const TcProduct &t1,
                                SkinnyTcArgs a1, const PairGeom &pg, uint8_t *ws, const WsLayout &L,
                                cudaStream_t st) {
  CUtensorMap m0[3], m1[3];
  const size_t part1 = L.partials + static_cast<size_t>(round_up(static_cast<int64_t>(pg.part0), 256));
  const size_t cnt1 = L.counters + static_cast<size_t>((a0.M + 127) / 128) * sizeof(uint32_t);
  if (!prepare_tc(t0, a0, ws, L.partials, L.counters, m0) || !prepare_tc(t1, a1, ws, part1, cnt1, m1))
    return QLORA_ERR_CUDA;
  const double flops = 2.0 * (a0.M * a0.C * a0.nq + a1.M * a1.C * a1.nq) * a0.R;
  const double bytes = 2.0 * (a0.M * a0.C + a1.M * a1.C);
  const bool pdl = g_trace.recs == nullptr;
  TraceScope ts(kid, flops, bytes, st);
  return launch_skinny_tc_pair(a0, m0, a1, m1, st, pdl) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
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

qlora_status qlora_quantize_nf4(const void *w_bf16, int64_t rows, int64_t cols, int32_t blocksize,
                                int32_t dq_block, const float codebook[16], qlora_nf4_weight *out, void *ws,
                                size_t ws_bytes, void *stream) {
  if (!w_bf16 || !codebook || !out || !out->codes || !out->scales || !out->c2) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
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
                                  tab, static_cast<uint32_t *>(ws), st, num_sms_current());
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
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
  if (!aligned16(x) || !aligned16(A) || !aligned16(B)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

qlora_status qlora_linear_fwd(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A, const void *B,
                              int32_t r, float s, void *y, void *ws, size_t ws_bytes, void *stream) {
  qlora_status cs = check_linear(x, T, qw, A, B, r, s);
  if (cs != QLORA_OK) return cs;
  if (T > 0 && !y) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(y)) return QLORA_ERR_MISALIGNED;
  const int64_t N = qw->rows, K = qw->cols;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < qlora_workspace_bytes(QLORA_OP_FWD, T, N, K, r))
    return QLORA_ERR_WORKSPACE;
  if (T == 0) return QLORA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const WsLayout L = ws_layout(QLORA_OP_FWD, T, N, K, r);
  const int64_t r64 = round_up(r, 64);
  uint16_t *su = reinterpret_cast<uint16_t *>(w8 + L.su_row);
  // sU = s X A^T [T, ceil64(r)]: the rank-r operand of the GEMV / GEMM
  if (decode_path(T, N)) {
    // a handful of rows: a latency-bound product, on a cluster kernel (one
    // wave, partial sums in distributed shared memory) where its slice fits
    const bool pdl = g_trace.recs == nullptr;
    if (lora_u_decode_smem_bytes(K, static_cast<int>(T)) <= kLoraUDecodeMaxSmem) {
      LoraUDecodeParams pu;
      pu.x = static_cast<const uint16_t *>(x);
      pu.A = static_cast<const uint16_t *>(A);
      pu.u = su;
      pu.K = K;
      pu.ldu = r64;
      pu.T = static_cast<int>(T);
      pu.r = r;
      pu.kc = 0;
      pu.alpha = s;
      {
        TraceScope ts(K_LORA_U, 2.0 * T * K * r, 2.0 * r * K, st);
        if (launch_lora_u_decode(pu, st, pdl) != cudaSuccess) return QLORA_ERR_CUDA;
      }
      return run_gemv(qw, x, T, su, r64, B, r, y, w8, L, st);
    }
    SkinnyParams pu = skinny_base(T, K, r, w8, L);
    pu.P = static_cast<const uint16_t *>(x);
    pu.ldp = K;
    pu.Q0 = static_cast<const uint16_t *>(A);
    pu.ldq = K;
    pu.alpha = s;
    pu.out0 = su;
    pu.out1 = nullptr;
    pu.ldo = r64;
    {
      TraceScope ts(K_LORA_U, 2.0 * T * K * r, 2.0 * T * K, st);
      if (launch_skinny(pu, false, false, OUT_HILO, st) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return run_gemv(qw, x, T, su, r64, B, r, y, w8, L, st);
  }
  SkinnyTcArgs au = tc_args(T, K, r, s);
  au.row_hi = su;
  au.ldo = r64;
  const TcProduct tu = {K_LORA_U, x, K, false, A, nullptr, K, false, geom_u(T, K, r)};
  qlora_status rs = run_skinny_tc(tu, au, w8, L, st);
  if (rs != QLORA_OK) return rs;
  return run_gemm(0, qw, x, su, r64, B, r, y, T, reinterpret_cast<uint32_t *>(ws), st);
}

qlora_status qlora_linear_bwd(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                              const void *B, int32_t r, float s, void *dx, void *dA, void *dB, void *ws,
                              size_t ws_bytes, void *stream) {
  qlora_status cs = check_linear(x, T, qw, A, B, r, s);
  if (cs != QLORA_OK) return cs;
  if ((T > 0 && (!dy || !dx)) || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(dx) || !aligned16(dA) || !aligned16(dB)) return QLORA_ERR_MISALIGNED;
  const int64_t N = qw->rows, K = qw->cols;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < qlora_workspace_bytes(QLORA_OP_BWD, T, N, K, r))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    // no tokens: the adapter gradients are empty sums
    if (cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 2, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const WsLayout L = ws_layout(QLORA_OP_BWD, T, N, K, r);
  const int64_t r64 = round_up(r, 64);
  const int64_t Tp = round_up(T, 8);
  auto plane = [&](size_t off) { return reinterpret_cast<uint16_t *>(w8 + off); };
  // TMA reads B in place for dU when its rows are a multiple of 16 bytes
  // (columns past r come back as zeros); otherwise B is first copied to
  // [N, ceil64(r)] rows.
  const void *bq = B;
  int64_t ldb = r;
  if (r % 8 != 0 || !aligned16(B)) {
    uint16_t *bpad = plane(L.bpad);
    if (launch_pad_cols(static_cast<const uint16_t *>(B), N, r, bpad, static_cast<int>(r64), st,
                        num_sms_current()) != cudaSuccess)
      return QLORA_ERR_CUDA;
    bq = bpad;
    ldb = r64;
  }
  // one grid: sU = s X A^T, transposed, as hi + lo planes [r, ceil8(T)]; and
  // dU = s dY B as a hi plane [T, ceil64(r)] for the dX GEMM plus transposed hi
  // + lo planes for dA
  const PairGeom g1 = geom_u_du(T, N, K, r);
  SkinnyTcArgs au = tc_args(T, K, r, s);
  au.t_hi = plane(L.suT_hi);
  au.t_lo = plane(L.suT_lo);
  au.ldt = Tp;
  SkinnyTcArgs ad = tc_args(T, N, r, s);
  ad.row_hi = plane(L.du_row);
  ad.ldo = r64;
  ad.t_hi = plane(L.duT_hi);
  ad.t_lo = plane(L.duT_lo);
  ad.ldt = Tp;
  const TcProduct tu = {K_LORA_U, x, K, false, A, nullptr, K, false, g1.g0};
  const TcProduct td = {K_LORA_DU, dy, N, false, bq, nullptr, ldb, true, g1.g1};
  qlora_status rs = run_skinny_tc_pair(K_LORA_U_DU, tu, au, td, ad, g1, w8, L, st);
  if (rs != QLORA_OK) return rs;
  // one grid: dB = dY^T (sU) [N, r] and dA = dU^T X [r, K]; it needs only the
  // planes above, so it runs on the side stream beside the dX GEMM (which
  // touches no other workspace than the status word) and joins before return
  const PairGeom g2 = geom_db_da(T, N, K, r);
  SkinnyTcArgs ab = tc_args(N, T, r, 1.0f);
  ab.row = static_cast<uint16_t *>(dB);
  SkinnyTcArgs aa = tc_args(K, T, r, 1.0f);
  aa.tr = static_cast<uint16_t *>(dA);
  const TcProduct tb = {K_LORA_DB, dy, N, true, plane(L.suT_hi), plane(L.suT_lo), Tp, false, g2.g0};
  const TcProduct ta = {K_LORA_DA, x, K, true, plane(L.duT_hi), plane(L.duT_lo), Tp, false, g2.g1};
  // (with a trace attached everything stays on the caller's stream, so that each
  // launch's events time that launch alone)
  SideStream *side = g_trace.recs == nullptr ? side_stream() : nullptr;
  if (side && cudaEventRecord(side->fork, st) != cudaSuccess) return QLORA_ERR_CUDA;
  // dX = dY W' + dU A, first in line for the SMs
  rs = run_gemm(1, qw, dy, plane(L.du_row), r64, A, r, dx, T, reinterpret_cast<uint32_t *>(ws), st);
  if (rs != QLORA_OK) return rs;
  if (!side) return run_skinny_tc_pair(K_LORA_DB_DA, tb, ab, ta, aa, g2, w8, L, st);
  if (cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess) return QLORA_ERR_CUDA;
  rs = run_skinny_tc_pair(K_LORA_DB_DA, tb, ab, ta, aa, g2, w8, L, side->s);
  if (cudaEventRecord(side->join, side->s) != cudaSuccess || cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return rs;
}

// ---------------------------------------------------------------------------
// Forward without a caller workspace.  Its scratch (status word, split
// counters, the U' planes and the split partial sums) lives in this fixed
// device array; each GPU that loads the library reserves it until exit.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

static void *noalloc_scratch_ptr() {
  // the symbol's device address, looked up once per device with that device current
  static void *ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

qlora_status qlora_linear_fwd_noalloc(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                      const void *B, int32_t r, float s, void *y, void *stream) {
  qlora_status cs = check_linear(x, T, qw, A, B, r, s);
  if (cs != QLORA_OK) return cs;
  const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, T, qw->rows, qw->cols, r);
  if (need == 0 || need > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_WORKSPACE;
  void *ws = noalloc_scratch_ptr();
  if (!ws) return QLORA_ERR_CUDA;
  // the status word and the split counters must start at zero
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes + kWsCounterBytes, st) != cudaSuccess) return QLORA_ERR_CUDA;
  return qlora_linear_fwd(x, T, qw, A, B, r, s, y, ws, QLORA_NOALLOC_SCRATCH_BYTES, stream);
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
