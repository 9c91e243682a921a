// Internal interfaces between the C-ABI layer and the kernel launchers.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

#include "sbsa.h"
#include <cuda_bf16.h>

namespace sbsa {

// One pooling job: x [n_heads, N, dim] -> centroids [n_heads/group, NB, dim]
// (+ radii [n_heads, NB] when rad != nullptr and group == 1).
struct PoolJob {
  const void* x;
  int n_heads;
  int group;
  float* cent;  // [n_heads/group, NB, dim] means, or nullptr when mm is set
  float* rad;
  float* mm;    // [n_heads, NB, 2, dim] coordinate-wise min then max, or nullptr
};

// Launch pooling of up to two jobs (same dtype and dim) as one grid.
cudaError_t launch_pool(int dtype, int dim, int seq_len, int block, const PoolJob* jobs,
                        int njobs, cudaStream_t stream);

struct SelectArgs {
  const float* qc;   // [Hs, NB, ds]
  const float* kc;   // [Hkv, NB, ds] centroids, or [Hkv, NB, 2, ds] min/max (minmax)
  const float* kr;   // [Hkv, NB] or nullptr
  int32_t* idx;      // [Hs, NB, kmax]
  int32_t* cnt;      // [Hs, NB]
  uint8_t* flags;    // [Hs, NB] or nullptr
  int n_sel_heads;   // Hs
  int kv_div;        // selection head hs scores against kv head hs / kv_div
  int nb;
  int ds;
  int kmax;
  int mode;          // SBSA_TOPK | SBSA_CUMMASS
  int minmax;        // 1: upper-bound scores from the min/max table
  // percentile gate (SBSA_GATE_PERCENTILE): pass 1 writes top-k lists and the
  // per-row cut margins, pass 2 rewrites the rows of fired tiles with top
  // rho*k; pass 0 is the ordinary single pass
  int pass;
  int rho;
  double* sigma;        // [Hs, NB] cut margins (NaN: no cut), written by pass 1
  const uint8_t* fire;  // [NB] 1 for fired tiles, read by pass 2
  const float* scores;  // [Hs, NB, NB] precomputed scores (centroid or row-max), or nullptr
  int top_k;
  float mass;
  int gate;
  float margin;
  int rescue;
  float tau;
  float score_scale;
  int* status;
};

// The percentile gate's tile decisions, in two halves so that the selection
// heads may be spread over several processes: the sum of each tile's margins
// over this call's Hs heads (head order), then -- once the sums cover every
// head -- the mean over total_heads and the floor(q T) smallest of the T tiles
// with more than k candidates.
cudaError_t launch_gate_sums(const double* sigma, double* sums, int n_sel_heads, int nb,
                             cudaStream_t stream);
cudaError_t launch_gate_fire(const double* sums, uint8_t* fire, int total_heads, int nb,
                             int top_k, float quantile, cudaStream_t stream);

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);

// Row-max tile scores: the fp32 centroids are split exactly into three bf16
// parts (c_parts), then scores[hs, i, j] = max over the tile's query rows (and
// the group's heads in group mode) of q_t . c_j * scale, for j < i.
struct RowmaxArgs {
  const void* q;           // [Hq, N, ds] bf16 (Q, or Q_idx in index mode)
  const float* c_f32;      // [Hkv, NB, ds]
  __nv_bfloat16* c_parts;  // [3, Hkv, NB, ds] scratch (hi, mid, lo planes)
  float* scores;         // [Hs, NB, NB]
  int hq, hkv, n, nb, ds, group_shared;
  float scale;
  int* status;
};
cudaError_t launch_rowmax(const RowmaxArgs& a, cudaStream_t stream);

// Whether the row-max kernel's shared memory (a 4-stage ring of part tiles,
// the query tile and the running maxima of NB candidates) fits one CTA.
bool rowmax_fits(int nb, int ds);

// Whether the selection kernel's shared memory holds at least two score rows
// of NB candidates (with the radii when the rescue branch is on).
bool select_fits(int nb, int ds, int rescue);

// Centroid block scores on the tensor cores: qc and kc are split into tf32
// hi / lo parts (scratch), then scores[hs, i, j] = qc[hs, i] . kc[hs / kv_div, j]
// * scale for j < i, to fp32 accuracy from three tf32 products.
struct CentroidScoreArgs {
  const float* qc;     // [Hs, NB, ds] pooled queries
  const float* kc;     // [Hkv, NB, ds] centroids
  float* q_hi;         // [Hs, NB, ds] scratch
  float* q_lo;         // [Hs, NB, ds] scratch
  float* c_hi;         // [Hkv, NB, ds] scratch
  float* c_lo;         // [Hkv, NB, ds] scratch
  float* scores;       // [Hs, NB, NB]
  int hs, hkv, kv_div, nb, ds;
  float scale;
  int* status;
};
cudaError_t launch_centroid_scores(const CentroidScoreArgs& a, cudaStream_t stream);

struct AttendArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  const int32_t* idx;
  const int32_t* cnt;
  int hq, hkv, n, d, block, dtype, group_shared, kmax;
  float sm_scale;
  int* status;
};

// Returns an SBSA_* code (SBSA_ERR_CUDA on launch/driver failure).  bf16
// with 128-token blocks runs the head-pair kernel for lists shared by a GQA
// group with an even number of query heads, else the persistent kernel; bf16
// with 64-token blocks runs the persistent kernel on two-block tiles; fp32
// runs the one-tile-per-CTA kernel.  The environment variable SBSA_ATTEND_KERNEL
// ("duo", "pair", "persistent", "single") overrides the choice where the
// requested kernel supports the arguments.
int launch_attend(const AttendArgs& a, cudaStream_t stream);

// The head-pair kernel (bf16, B = 128, d in {64, 128}, even group size).
int launch_attend_pair(const AttendArgs& a, cudaStream_t stream);

// The one-tile-per-CTA kernel (every supported dtype / block / d).
int launch_attend_single(const AttendArgs& a, cudaStream_t stream);

// The persistent pipelined kernel (bf16, B = 128, d in {64, 128}).
int launch_attend_persistent(const AttendArgs& a, cudaStream_t stream);
// exp2_fma (the FMA-pipe exponential the persistent kernel can use for a
// part of its softmax) applied to n floats in device memory.
cudaError_t launch_exp2_fma(const float* x, float* y, long long n, cudaStream_t stream);

// The persistent pipelined kernel on tiles of two 64-token query blocks
// (bf16, B = 64, d in {64, 128}).
int launch_attend_persistent64(const AttendArgs& a, cudaStream_t stream);

// Two independent query tiles per CTA (bf16, B = 128, d in {64, 128}, one
// list per query head).
int launch_attend_duo(const AttendArgs& a, cudaStream_t stream);

// One CTA waiting on an mbarrier that never completes, through the bounded
// wait of the pipelines; records SBSA_ERR_TIMEOUT when the limit expires.
cudaError_t launch_wait_probe(uint64_t timeout_ns, int* status, cudaStream_t stream);

// Device status word of the current device (recorded by kernels).
int* device_status_ptr();

// The argument checks every entry point makes (SBSA_OK or an error code).
int validate_params(const sbsa_params* p);

}  // namespace sbsa
