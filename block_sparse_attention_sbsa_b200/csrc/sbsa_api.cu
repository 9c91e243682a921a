// C-ABI entry points: argument validation (before any launch), workspace
// carving, dispatch to the pooling / selection / attention launchers, and
// the per-device status word that kernels use to report runtime errors.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"

// Written by kernels (first error wins), read and cleared by sbsa_get_status.
__device__ int g_sbsa_device_status = 0;

namespace sbsa {

int* device_status_ptr() {
  static std::mutex mu;
  static int* cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_sbsa_device_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(ptr);
  }
  return cache[dev];
}

namespace {

struct Derived {
  int nb;           // number of blocks
  int group;        // Hq / Hkv
  int hs;           // selection heads
  int ds;           // score dimension
  int need_kmax;    // smallest valid max_blocks
  float sm_scale;
  float score_scale;
};

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shape/option checks shared by every entry point.
int validate(const sbsa_params* p, Derived* d) {
  if (!p) return SBSA_ERR_INVALID_ARG;
  if (p->n_q_heads < 1 || p->n_kv_heads < 1 || p->n_q_heads % p->n_kv_heads != 0)
    return SBSA_ERR_INVALID_ARG;
  if (p->seq_len < 1) return SBSA_ERR_INVALID_ARG;
  if (p->dtype != SBSA_BF16 && p->dtype != SBSA_FP32) return SBSA_ERR_INVALID_ARG;
  if (p->head_dim <= 0 || p->block_size <= 0 || p->index_dim < 0) return SBSA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return SBSA_ERR_UNSUPPORTED;
  if (p->block_size != 64 && p->block_size != 128) return SBSA_ERR_UNSUPPORTED;
  if (p->index_dim != 0 && p->index_dim != 64 && p->index_dim != 128) return SBSA_ERR_UNSUPPORTED;
  if (p->select_mode != SBSA_TOPK && p->select_mode != SBSA_CUMMASS) return SBSA_ERR_INVALID_ARG;
  if (p->select_mode == SBSA_TOPK && p->top_k < 1) return SBSA_ERR_INVALID_ARG;
  if (p->select_mode == SBSA_CUMMASS &&
      !(p->mass_threshold > 0.f && p->mass_threshold <= 1.f))
    return SBSA_ERR_INVALID_ARG;
  if (p->gate != 0 && p->gate != SBSA_GATE_GAP && p->gate != SBSA_GATE_PERCENTILE)
    return SBSA_ERR_INVALID_ARG;
  if (p->gate && p->select_mode != SBSA_TOPK) return SBSA_ERR_INVALID_ARG;
  if (p->gate == SBSA_GATE_GAP && !(p->gate_margin >= 0.f && std::isfinite(p->gate_margin)))
    return SBSA_ERR_INVALID_ARG;
  if (p->gate == SBSA_GATE_PERCENTILE &&
      (!(p->gate_quantile >= 0.f && p->gate_quantile <= 1.f) || p->gate_rho < 1))
    return SBSA_ERR_INVALID_ARG;
  if (p->rescue && std::isnan(p->rescue_tau)) return SBSA_ERR_INVALID_ARG;
  if (p->backbone != SBSA_BACKBONE_MEAN && p->backbone != SBSA_BACKBONE_MINMAX)
    return SBSA_ERR_INVALID_ARG;
  if (p->backbone == SBSA_BACKBONE_MINMAX && p->rescue) return SBSA_ERR_INVALID_ARG;
  if (p->tile_score != SBSA_TILE_MEAN && p->tile_score != SBSA_TILE_ROWMAX)
    return SBSA_ERR_INVALID_ARG;
  if (p->tile_score == SBSA_TILE_ROWMAX &&
      (p->backbone != SBSA_BACKBONE_MEAN || p->rescue || p->dtype != SBSA_BF16))
    return SBSA_ERR_INVALID_ARG;
  if (!(p->sm_scale >= 0.f) || !std::isfinite(p->sm_scale)) return SBSA_ERR_INVALID_ARG;
  if (!(p->score_scale >= 0.f) || !std::isfinite(p->score_scale)) return SBSA_ERR_INVALID_ARG;
  Derived o;
  o.nb = (p->seq_len + p->block_size - 1) / p->block_size;
  o.group = p->n_q_heads / p->n_kv_heads;
  o.hs = p->group_shared ? p->n_kv_heads : p->n_q_heads;
  o.ds = p->index_dim ? p->index_dim : p->head_dim;
  if (p->select_mode == SBSA_CUMMASS || p->rescue) {
    o.need_kmax = o.nb;
  } else {
    long long budget = p->top_k;
    if (p->gate == SBSA_GATE_GAP) budget = 2LL * p->top_k;
    if (p->gate == SBSA_GATE_PERCENTILE) budget = (long long)p->gate_rho * p->top_k;
    if (budget > o.nb - 1) budget = o.nb - 1;
    o.need_kmax = (int)budget + 1;
  }
  if (p->max_blocks < o.need_kmax) return SBSA_ERR_INVALID_ARG;
  if ((long long)p->n_q_heads * o.nb > 0x7FFFFFFFLL) return SBSA_ERR_UNSUPPORTED;
  // the percentile gate's tile means are held in one CTA's shared memory
  if (p->gate == SBSA_GATE_PERCENTILE && (size_t)o.nb * sizeof(double) > 227 * 1024)
    return SBSA_ERR_UNSUPPORTED;
  // the selection kernel holds at least two score rows in shared memory, the
  // row-max kernel the running maxima of a tile's candidates
  if (!select_fits(o.nb, o.ds, p->rescue ? 1 : 0)) return SBSA_ERR_UNSUPPORTED;
  if (p->tile_score == SBSA_TILE_ROWMAX && !rowmax_fits(o.nb, o.ds)) return SBSA_ERR_UNSUPPORTED;
  o.sm_scale = p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt((float)p->head_dim);
  o.score_scale = p->score_scale > 0.f ? p->score_scale : 1.0f / std::sqrt((float)o.ds);
  if (d) *d = o;
  return SBSA_OK;
}

}  // namespace

int validate_params(const sbsa_params* p) { return validate(p, nullptr); }

namespace {

int attend_supported(const sbsa_params* p) {
  if (p->dtype == SBSA_FP32 && !(p->head_dim == 64 && p->block_size == 64))
    return SBSA_ERR_UNSUPPORTED;
  return SBSA_OK;
}

// Centroid scores run as a tensor-core product (with the mean backbone and
// mean tile scores) wherever a workspace holds their scratch.
bool centroid_tc(const sbsa_params* p) {
  return p->backbone == SBSA_BACKBONE_MEAN && p->tile_score == SBSA_TILE_MEAN;
}

// Scratch of a precomputed score table, placed from offset `off`: for the
// row-max tile scores the three bf16 parts of the centroids, for the tensor-core centroid
// scores the tf32 hi / lo parts of the pooled queries and the centroids;
// then the table [Hs, NB, NB].
struct ScoreScratch {
  size_t cbf, q_hi, q_lo, c_hi, c_lo, scores;
};

size_t score_scratch(const sbsa_params* p, const Derived& d, size_t off, ScoreScratch* o) {
  const bool rowmax = p->tile_score == SBSA_TILE_ROWMAX;
  const bool tc = centroid_tc(p);
  const size_t q_bytes = (size_t)d.hs * d.nb * d.ds * 4;
  const size_t c_bytes = (size_t)p->n_kv_heads * d.nb * d.ds * 4;
  o->cbf = off;
  if (rowmax) off = round_up(off + 3 * (c_bytes / 2), 256);
  o->q_hi = off;
  if (tc) off = round_up(off + q_bytes, 256);
  o->q_lo = off;
  if (tc) off = round_up(off + q_bytes, 256);
  o->c_hi = off;
  if (tc) off = round_up(off + c_bytes, 256);
  o->c_lo = off;
  if (tc) off = round_up(off + c_bytes, 256);
  o->scores = off;
  if (rowmax || tc) off = round_up(off + (size_t)d.hs * d.nb * d.nb * 4, 256);
  return off;
}

struct GateScratch {
  size_t sigma, sums, fire;
};

struct WsLayout {
  size_t qc, kc, kr, idx, cnt, flags, total;
  GateScratch gs;
  ScoreScratch sc;
};

// Scratch of the percentile gate, placed from offset `off`: per-row margins
// (double), per-tile margin sums (double) and per-tile decisions.
size_t gate_scratch(const sbsa_params* p, const Derived& d, size_t off, GateScratch* g) {
  const bool on = p->gate == SBSA_GATE_PERCENTILE;
  g->sigma = off;
  if (on) off = round_up(off + (size_t)d.hs * d.nb * 8, 256);
  g->sums = off;
  if (on) off = round_up(off + (size_t)d.nb * 8, 256);
  g->fire = off;
  if (on) off = round_up(off + (size_t)d.nb, 256);
  return off;
}

WsLayout layout(const sbsa_params* p, const Derived& d, bool lists) {
  WsLayout w{};
  size_t off = 0;
  w.qc = off;
  off = round_up(off + (size_t)d.hs * d.nb * d.ds * 4, 256);
  w.kc = off;
  const size_t tables_per_block = p->backbone == SBSA_BACKBONE_MINMAX ? 2 : 1;
  off = round_up(off + tables_per_block * p->n_kv_heads * d.nb * d.ds * 4, 256);
  w.kr = off;
  off = round_up(off + (p->rescue ? (size_t)p->n_kv_heads * d.nb * 4 : 0), 256);
  w.idx = off;
  off = round_up(off + (lists ? (size_t)d.hs * d.nb * p->max_blocks * 4 : 0), 256);
  w.cnt = off;
  off = round_up(off + (lists ? (size_t)d.hs * d.nb * 4 : 0), 256);
  w.flags = off;
  off = round_up(off + (lists ? (size_t)d.hs * d.nb : 0), 256);
  off = gate_scratch(p, d, off, &w.gs);
  off = score_scratch(p, d, off, &w.sc);
  w.total = off;
  return w;
}

int cuda_code(cudaError_t e) { return e == cudaSuccess ? SBSA_OK : SBSA_ERR_CUDA; }

SelectArgs select_args(const sbsa_params* p, const Derived& d, const float* qc, const float* kc,
                       const float* kr, int32_t* idx, int32_t* cnt, uint8_t* flags) {
  SelectArgs a{};
  a.qc = qc;
  a.kc = kc;
  a.kr = kr;
  a.idx = idx;
  a.cnt = cnt;
  a.flags = flags;
  a.n_sel_heads = d.hs;
  a.kv_div = p->group_shared ? 1 : d.group;
  a.nb = d.nb;
  a.ds = d.ds;
  a.kmax = p->max_blocks;
  a.mode = p->select_mode;
  a.minmax = p->backbone == SBSA_BACKBONE_MINMAX ? 1 : 0;
  a.top_k = p->top_k;
  a.mass = p->mass_threshold;
  a.gate = p->gate == SBSA_GATE_GAP ? 1 : 0;
  a.rho = p->gate_rho;
  a.margin = p->gate_margin;
  a.rescue = p->rescue ? 1 : 0;
  a.tau = p->rescue_tau;
  a.score_scale = d.score_scale;
  a.status = device_status_ptr();
  return a;
}

CentroidScoreArgs centroid_args(const sbsa_params* p, const Derived& d, const float* qc,
                                const float* kc, unsigned char* scratch, const ScoreScratch& o,
                                float* scores) {
  CentroidScoreArgs a{};
  a.qc = qc;
  a.kc = kc;
  a.q_hi = reinterpret_cast<float*>(scratch + o.q_hi);
  a.q_lo = reinterpret_cast<float*>(scratch + o.q_lo);
  a.c_hi = reinterpret_cast<float*>(scratch + o.c_hi);
  a.c_lo = reinterpret_cast<float*>(scratch + o.c_lo);
  a.scores = scores;
  a.hs = d.hs;
  a.hkv = p->n_kv_heads;
  a.kv_div = p->group_shared ? 1 : d.group;
  a.nb = d.nb;
  a.ds = d.ds;
  a.scale = d.score_scale;
  a.status = device_status_ptr();
  return a;
}

// The percentile gate's first pass: top-k lists and per-row margins, then
// the per-tile sums of the margins over this call's heads into `sums`.
int gate_first(const Derived& d, SelectArgs a, unsigned char* scratch, const GateScratch& g,
               double* sums, cudaStream_t s) {
  a.sigma = reinterpret_cast<double*>(scratch + g.sigma);
  a.fire = scratch + g.fire;
  a.pass = 1;
  int rc = cuda_code(launch_select(a, s));
  if (rc) return rc;
  return cuda_code(launch_gate_sums(a.sigma, sums, d.hs, d.nb, s));
}

// Its second pass: the tile decisions from sums that cover `total_heads`
// heads, then top rho*k in the rows of the fired tiles.
int gate_second(const sbsa_params* p, const Derived& d, SelectArgs a, unsigned char* scratch,
                const GateScratch& g, const double* sums, int total_heads, cudaStream_t s) {
  uint8_t* fire = scratch + g.fire;
  a.sigma = reinterpret_cast<double*>(scratch + g.sigma);
  a.fire = fire;
  int rc = cuda_code(
      launch_gate_fire(sums, fire, total_heads, d.nb, p->top_k, p->gate_quantile, s));
  if (rc) return rc;
  a.pass = 2;
  return cuda_code(launch_select(a, s));
}

// The selection on a stream: one launch, or for the percentile gate its
// four (top-k lists and margins, per-tile sums, tile decisions, fired tiles
// again).
int run_select(const sbsa_params* p, const Derived& d, SelectArgs a, unsigned char* scratch,
               const GateScratch& g, cudaStream_t s) {
  if (p->gate != SBSA_GATE_PERCENTILE) return cuda_code(launch_select(a, s));
  double* sums = reinterpret_cast<double*>(scratch + g.sums);
  int rc = gate_first(d, a, scratch, g, sums, s);
  if (rc) return rc;
  return gate_second(p, d, a, scratch, g, sums, d.hs, s);
}

AttendArgs attend_args(const sbsa_params* p, const Derived& d, const void* q, const void* k,
                       const void* v, const int32_t* idx, const int32_t* cnt, void* o) {
  AttendArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.idx = idx;
  a.cnt = cnt;
  a.hq = p->n_q_heads;
  a.hkv = p->n_kv_heads;
  a.n = p->seq_len;
  a.d = p->head_dim;
  a.block = p->block_size;
  a.dtype = p->dtype;
  a.group_shared = p->group_shared ? 1 : 0;
  a.kmax = p->max_blocks;
  a.sm_scale = d.sm_scale;
  a.status = device_status_ptr();
  return a;
}

}  // namespace
}  // namespace sbsa

using namespace sbsa;

extern "C" {

int sbsa_version(void) { return 104; }

const char* sbsa_status_string(int code) {
  switch (code) {
    case SBSA_OK: return "ok";
    case SBSA_ERR_INVALID_ARG: return "invalid argument";
    case SBSA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SBSA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case SBSA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case SBSA_ERR_TIMEOUT: return "a kernel wait timed out";
    case SBSA_ERR_DEVICE: return "a kernel met an out-of-range list entry";
    default: return "unknown status";
  }
}

int sbsa_pool_blocks(const sbsa_params* p, const void* x, int n_heads, int dim, int group,
                     float* centroids, float* radii, void* stream) {
  if (!p || !x || !centroids) return SBSA_ERR_INVALID_ARG;
  if (p->seq_len < 1 || p->block_size <= 0) return SBSA_ERR_INVALID_ARG;
  if (p->dtype != SBSA_BF16 && p->dtype != SBSA_FP32) return SBSA_ERR_INVALID_ARG;
  if (p->block_size != 64 && p->block_size != 128) return SBSA_ERR_UNSUPPORTED;
  if (n_heads < 1 || group < 1 || n_heads % group != 0) return SBSA_ERR_INVALID_ARG;
  if (dim != 64 && dim != 128) return SBSA_ERR_UNSUPPORTED;
  if (radii && group != 1) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(x)) return SBSA_ERR_INVALID_ARG;
  PoolJob job{x, n_heads, group, centroids, radii, nullptr};
  return cuda_code(launch_pool(p->dtype, dim, p->seq_len, p->block_size, &job, 1,
                               static_cast<cudaStream_t>(stream)));
}

int sbsa_pool_minmax(const sbsa_params* p, const void* x, int n_heads, int dim, float* minmax,
                     void* stream) {
  if (!p || !x || !minmax) return SBSA_ERR_INVALID_ARG;
  if (p->seq_len < 1 || p->block_size <= 0) return SBSA_ERR_INVALID_ARG;
  if (p->dtype != SBSA_BF16 && p->dtype != SBSA_FP32) return SBSA_ERR_INVALID_ARG;
  if (p->block_size != 64 && p->block_size != 128) return SBSA_ERR_UNSUPPORTED;
  if (n_heads < 1) return SBSA_ERR_INVALID_ARG;
  if (dim != 64 && dim != 128) return SBSA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(minmax)) return SBSA_ERR_INVALID_ARG;
  PoolJob job{x, n_heads, 1, nullptr, nullptr, minmax};
  return cuda_code(launch_pool(p->dtype, dim, p->seq_len, p->block_size, &job, 1,
                               static_cast<cudaStream_t>(stream)));
}

int sbsa_select(const sbsa_params* p, const float* q_cent, const float* k_cent,
                const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (!q_cent || !k_cent || !idx || !cnt) return SBSA_ERR_INVALID_ARG;
  if (p->rescue && !k_radius) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(q_cent) || !aligned16(k_cent)) return SBSA_ERR_INVALID_ARG;
  if (p->gate == SBSA_GATE_PERCENTILE) return SBSA_ERR_WORKSPACE;  // use sbsa_select_ws
  SelectArgs a = select_args(p, d, q_cent, k_cent, p->rescue ? k_radius : nullptr, idx, cnt,
                             flags);
  return cuda_code(launch_select(a, static_cast<cudaStream_t>(stream)));
}

size_t sbsa_select_workspace_bytes(const sbsa_params* p) {
  Derived d;
  if (validate(p, &d) != SBSA_OK) return 0;
  GateScratch g;
  ScoreScratch sc;
  const size_t off = gate_scratch(p, d, 0, &g);
  return centroid_tc(p) ? score_scratch(p, d, off, &sc) : off;
}

size_t sbsa_score_centroids_workspace_bytes(const sbsa_params* p) {
  Derived d;
  if (validate(p, &d) != SBSA_OK || !centroid_tc(p)) return 0;
  ScoreScratch sc;
  score_scratch(p, d, 0, &sc);
  return sc.scores;  // the split parts; the table is the caller's
}

int sbsa_score_centroids(const sbsa_params* p, const float* q_cent, const float* k_cent,
                         float* scores, void* workspace, size_t ws_bytes, void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (!centroid_tc(p)) return SBSA_ERR_UNSUPPORTED;
  if (!q_cent || !k_cent || !scores) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(q_cent) || !aligned16(k_cent) || !aligned16(scores)) return SBSA_ERR_INVALID_ARG;
  const size_t need = sbsa_score_centroids_workspace_bytes(p);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < need)
    return SBSA_ERR_WORKSPACE;
  ScoreScratch sc;
  score_scratch(p, d, 0, &sc);
  return cuda_code(launch_centroid_scores(
      centroid_args(p, d, q_cent, k_cent, static_cast<unsigned char*>(workspace), sc, scores),
      static_cast<cudaStream_t>(stream)));
}

size_t sbsa_score_rowmax_workspace_bytes(const sbsa_params* p) {
  Derived d;
  if (validate(p, &d) != SBSA_OK || p->tile_score != SBSA_TILE_ROWMAX) return 0;
  return round_up(3 * (size_t)p->n_kv_heads * d.nb * d.ds * 2, 256);
}

namespace {
RowmaxArgs rowmax_args(const sbsa_params* p, const Derived& d, const void* q_src,
                       const float* k_cent, void* c_parts, float* scores) {
  RowmaxArgs a{};
  a.q = q_src;
  a.c_f32 = k_cent;
  a.c_parts = static_cast<__nv_bfloat16*>(c_parts);
  a.scores = scores;
  a.hq = p->n_q_heads;
  a.hkv = p->n_kv_heads;
  a.n = p->seq_len;
  a.nb = d.nb;
  a.ds = d.ds;
  a.group_shared = p->group_shared ? 1 : 0;
  a.scale = d.score_scale;
  a.status = device_status_ptr();
  return a;
}
}  // namespace

int sbsa_score_rowmax(const sbsa_params* p, const void* q_src, const float* k_cent,
                      float* scores, void* workspace, size_t ws_bytes, void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (p->tile_score != SBSA_TILE_ROWMAX) return SBSA_ERR_UNSUPPORTED;
  if (!q_src || !k_cent || !scores) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(q_src) || !aligned16(k_cent) || !aligned16(scores)) return SBSA_ERR_INVALID_ARG;
  const size_t need = sbsa_score_rowmax_workspace_bytes(p);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < need)
    return SBSA_ERR_WORKSPACE;
  return cuda_code(launch_rowmax(rowmax_args(p, d, q_src, k_cent, workspace, scores),
                                 static_cast<cudaStream_t>(stream)));
}

int sbsa_select_scores(const sbsa_params* p, const float* scores, int32_t* idx, int32_t* cnt,
                       uint8_t* flags, void* workspace, size_t ws_bytes, void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (!scores || !idx || !cnt) return SBSA_ERR_INVALID_ARG;
  if (p->rescue) return SBSA_ERR_INVALID_ARG;  // the rescue bound needs the tables
  GateScratch g;
  const size_t need = gate_scratch(p, d, 0, &g);
  if (need && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
               ws_bytes < need))
    return SBSA_ERR_WORKSPACE;
  SelectArgs a = select_args(p, d, nullptr, nullptr, nullptr, idx, cnt, flags);
  a.scores = scores;
  return run_select(p, d, a, static_cast<unsigned char*>(workspace), g,
                    static_cast<cudaStream_t>(stream));
}

namespace {
// Checks and scores shared by sbsa_select_ws and the two halves of the
// percentile gate: validates the arguments and the workspace, takes the
// tensor-core centroid scores into it where they apply, and returns the
// selection's arguments (rc != SBSA_OK: nothing was launched).
struct SelectWs {
  int rc;
  Derived d;
  GateScratch g;
  SelectArgs a;
};

SelectWs select_ws_prepare(const sbsa_params* p, const float* q_cent, const float* k_cent,
                           const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                           void* workspace, size_t ws_bytes, bool scores_now,
                           cudaStream_t s) {
  SelectWs r{};
  r.rc = validate(p, &r.d);
  if (r.rc) return r;
  const Derived& d = r.d;
  r.rc = SBSA_ERR_INVALID_ARG;
  if (!q_cent || !k_cent || !idx || !cnt) return r;
  if (p->rescue && !k_radius) return r;
  if (!aligned16(q_cent) || !aligned16(k_cent)) return r;
  // workspace: the percentile gate's scratch, then the score table's
  ScoreScratch sc;
  const size_t gate_end = gate_scratch(p, d, 0, &r.g);
  const size_t need = centroid_tc(p) ? score_scratch(p, d, gate_end, &sc) : gate_end;
  r.rc = SBSA_ERR_WORKSPACE;
  if (need && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
               ws_bytes < need))
    return r;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  r.a = select_args(p, d, q_cent, k_cent, p->rescue ? k_radius : nullptr, idx, cnt, flags);
  r.rc = SBSA_OK;
  if (centroid_tc(p)) {
    float* scores = reinterpret_cast<float*>(ws + sc.scores);
    if (scores_now)
      r.rc = cuda_code(launch_centroid_scores(centroid_args(p, d, q_cent, k_cent, ws, sc, scores), s));
    r.a.scores = scores;  // the pooled queries stay for the rescue bound
  }
  return r;
}
}  // namespace

int sbsa_select_ws(const sbsa_params* p, const float* q_cent, const float* k_cent,
                   const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                   void* workspace, size_t ws_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SelectWs r = select_ws_prepare(p, q_cent, k_cent, k_radius, idx, cnt, flags, workspace,
                                 ws_bytes, true, s);
  if (r.rc) return r.rc;
  return run_select(p, r.d, r.a, static_cast<unsigned char*>(workspace), r.g, s);
}

int sbsa_select_gate_partial(const sbsa_params* p, const float* q_cent, const float* k_cent,
                             const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                             void* workspace, size_t ws_bytes, double* tile_sums,
                             void* stream) {
  const int rc = validate(p, nullptr);
  if (rc) return rc;
  if (p->gate != SBSA_GATE_PERCENTILE || p->tile_score != SBSA_TILE_MEAN)
    return SBSA_ERR_INVALID_ARG;
  if (!tile_sums || (reinterpret_cast<uintptr_t>(tile_sums) & 7u) != 0)
    return SBSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SelectWs r = select_ws_prepare(p, q_cent, k_cent, k_radius, idx, cnt, flags, workspace,
                                 ws_bytes, true, s);
  if (r.rc) return r.rc;
  return gate_first(r.d, r.a, static_cast<unsigned char*>(workspace), r.g, tile_sums, s);
}

int sbsa_select_gate_finish(const sbsa_params* p, const float* q_cent, const float* k_cent,
                            const float* k_radius, int32_t* idx, int32_t* cnt, uint8_t* flags,
                            void* workspace, size_t ws_bytes, const double* tile_sums,
                            int total_heads, void* stream) {
  const int rc = validate(p, nullptr);
  if (rc) return rc;
  if (p->gate != SBSA_GATE_PERCENTILE || p->tile_score != SBSA_TILE_MEAN)
    return SBSA_ERR_INVALID_ARG;
  if (!tile_sums || (reinterpret_cast<uintptr_t>(tile_sums) & 7u) != 0)
    return SBSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SelectWs r = select_ws_prepare(p, q_cent, k_cent, k_radius, idx, cnt, flags, workspace,
                                 ws_bytes, false, s);
  if (r.rc) return r.rc;
  if (total_heads < r.d.hs) return SBSA_ERR_INVALID_ARG;
  return gate_second(p, r.d, r.a, static_cast<unsigned char*>(workspace), r.g, tile_sums,
                     total_heads, s);
}

int sbsa_attend(const sbsa_params* p, const void* q, const void* k, const void* v,
                const int32_t* idx, const int32_t* cnt, void* o, void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (!q || !k || !v || !idx || !cnt || !o) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SBSA_ERR_INVALID_ARG;
  rc = attend_supported(p);
  if (rc) return rc;
  return launch_attend(attend_args(p, d, q, k, v, idx, cnt, o), static_cast<cudaStream_t>(stream));
}

size_t sbsa_prefill_workspace_bytes(const sbsa_params* p) {
  Derived d;
  if (validate(p, &d) != SBSA_OK) return 0;
  return layout(p, d, true).total;
}

int sbsa_prefill(const sbsa_params* p, const void* q, const void* k, const void* v,
                 const void* q_idx, const void* k_idx, void* o, void* workspace,
                 size_t ws_bytes, int32_t* idx_out, int32_t* cnt_out, uint8_t* flags_out,
                 void* stream) {
  Derived d;
  int rc = validate(p, &d);
  if (rc) return rc;
  if (!q || !k || !v || !o) return SBSA_ERR_INVALID_ARG;
  if (p->index_dim && (!q_idx || !k_idx)) return SBSA_ERR_INVALID_ARG;
  if ((idx_out == nullptr) != (cnt_out == nullptr)) return SBSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SBSA_ERR_INVALID_ARG;
  if (p->index_dim && (!aligned16(q_idx) || !aligned16(k_idx))) return SBSA_ERR_INVALID_ARG;
  rc = attend_supported(p);
  if (rc) return rc;
  const bool lists_in_ws = idx_out == nullptr;
  WsLayout w = layout(p, d, lists_in_ws);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < w.total)
    return SBSA_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* qc = reinterpret_cast<float*>(ws + w.qc);
  float* kc = reinterpret_cast<float*>(ws + w.kc);
  float* kr = p->rescue ? reinterpret_cast<float*>(ws + w.kr) : nullptr;
  int32_t* idx = lists_in_ws ? reinterpret_cast<int32_t*>(ws + w.idx) : idx_out;
  int32_t* cnt = lists_in_ws ? reinterpret_cast<int32_t*>(ws + w.cnt) : cnt_out;
  uint8_t* flags = flags_out ? flags_out
                             : (lists_in_ws ? reinterpret_cast<uint8_t*>(ws + w.flags) : nullptr);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* xs_k = p->index_dim ? k_idx : k;
  const void* xs_q = p->index_dim ? q_idx : q;
  const bool minmax = p->backbone == SBSA_BACKBONE_MINMAX;
  PoolJob jobs[2] = {
      {xs_k, p->n_kv_heads, 1, minmax ? nullptr : kc, kr, minmax ? kc : nullptr},
      {xs_q, p->n_q_heads, p->group_shared ? d.group : 1, qc, nullptr, nullptr},
  };
  // row-max tile scores read the query rows themselves: no pooled queries
  const bool rowmax = p->tile_score == SBSA_TILE_ROWMAX;
  rc = cuda_code(launch_pool(p->dtype, d.ds, p->seq_len, p->block_size, jobs, rowmax ? 1 : 2, s));
  if (rc) return rc;
  SelectArgs sa = select_args(p, d, qc, kc, kr, idx, cnt, flags);
  float* scores = reinterpret_cast<float*>(ws + w.sc.scores);
  if (p->tile_score == SBSA_TILE_ROWMAX) {
    rc = cuda_code(launch_rowmax(rowmax_args(p, d, xs_q, kc, ws + w.sc.cbf, scores), s));
    if (rc) return rc;
    sa.scores = scores;
    sa.qc = nullptr;
  } else if (centroid_tc(p)) {
    rc = cuda_code(launch_centroid_scores(centroid_args(p, d, qc, kc, ws, w.sc, scores), s));
    if (rc) return rc;
    sa.scores = scores;  // the pooled queries stay for the rescue bound
  }
  rc = run_select(p, d, sa, ws, w.gs, s);
  if (rc) return rc;
  return launch_attend(attend_args(p, d, q, k, v, idx, cnt, o), s);
}

int sbsa_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000ull) timeout_ns = 1000ull;
  if (timeout_ns > 10000000000ull) timeout_ns = 10000000000ull;
  return cuda_code(launch_wait_probe(timeout_ns, device_status_ptr(),
                                     static_cast<cudaStream_t>(stream)));
}

int sbsa_exp2_fma_eval(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return SBSA_ERR_INVALID_ARG;
  if (n == 0) return SBSA_OK;
  if (!x || !y) return SBSA_ERR_INVALID_ARG;
  return cuda_code(launch_exp2_fma(x, y, (long long)n, static_cast<cudaStream_t>(stream)));
}

int sbsa_get_status(void* stream, int* device_status) {
  if (!device_status) return SBSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SBSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_sbsa_device_status, sizeof(int)) != cudaSuccess)
    return SBSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_sbsa_device_status, &zero, sizeof(int)) != cudaSuccess)
    return SBSA_ERR_CUDA;
  *device_status = v;
  return SBSA_OK;
}

}  // extern "C"
