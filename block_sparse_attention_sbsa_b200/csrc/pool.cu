// Block pooling: centroid (mean of a block's rows) and radius (largest l2
// distance of a row from the centroid), optionally averaged over a group of
// consecutive heads; or the coordinate-wise minimum and maximum of a block's
// rows (the K-min / K-max table of the upper-bound scoring backbone).
//
// "RBS-Attention" (iaonda.com), method paragraph: key blocks are summarised
// by a centroid and a dynamic, prompt/layer/head-dependent key-block radius.
// "Uncertainty-gated selection for block-sparse attention", Metodologia
// step 1: mean pooling of key blocks (SSA-style K-mean); step 2: selection
// per query tile.  "MiniMax presenta MSA": one selection per GQA group.
//
// HBM-bound: every element of x is read exactly once with 16-byte vector
// loads; a CTA owns one (output head, block) pair.  When the radius is
// wanted the block stays in registers between the mean and the distance pass.
#include <cuda_bf16.h>

#include "internal.h"

namespace sbsa {
namespace {

constexpr int kPoolThreads = 256;

struct PoolGrid {
  PoolJob job[2];
  int nctas0;  // CTAs of job 0; the rest belong to job 1
  int nb;
  int n;
  int block;
};

template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void to_float(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct Vec16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void to_float(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T, int DIM>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __grid_constant__ PoolGrid g) {
  constexpr int E = Vec16<T>::E;
  constexpr int VPR = DIM / E;             // 16-byte vectors per row
  constexpr int RPP = kPoolThreads / VPR;  // rows covered by one pass of the CTA
  constexpr int MAXP = (128 + RPP - 1) / RPP;
  static_assert(VPR <= 32 && 32 % VPR == 0, "row must map onto a lane group");

  __shared__ float red[RPP][DIM];
  __shared__ float cs[DIM];
  __shared__ float wmax[kPoolThreads / 32];

  int b = blockIdx.x;
  const bool second = b >= g.nctas0;
  const PoolJob job = second ? g.job[1] : g.job[0];
  if (second) b -= g.nctas0;
  const int j = b % g.nb;
  const int hs = b / g.nb;
  const int row0 = j * g.block;
  const int nrows = min(g.block, g.n - row0);
  const int tid = threadIdx.x;
  const int vec = tid % VPR;
  const int rsub = tid / VPR;
  const bool want_r = job.rad != nullptr;

  if (job.mm) {
    // coordinate-wise minimum and maximum over the block's rows
    float mn[E], mx[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      mn[e] = INFINITY;
      mx[e] = -INFINITY;
    }
    const T* base = static_cast<const T*>(job.x) + ((size_t)hs * g.n + row0) * DIM + vec * E;
    for (int r = rsub; r < nrows; r += RPP) {
      float f[E];
      Vec16<T>::to_float(ld_stream(base + (size_t)r * DIM), f);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        mn[e] = fminf(mn[e], f[e]);
        mx[e] = fmaxf(mx[e], f[e]);
      }
    }
    float* out = job.mm + ((size_t)hs * g.nb + j) * 2 * DIM;
#pragma unroll
    for (int e = 0; e < E; ++e) red[rsub][vec * E + e] = mn[e];
    __syncthreads();
    for (int col = tid; col < DIM; col += kPoolThreads) {
      float m = red[0][col];
      for (int r = 1; r < RPP; ++r) m = fminf(m, red[r][col]);
      out[col] = m;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) red[rsub][vec * E + e] = mx[e];
    __syncthreads();
    for (int col = tid; col < DIM; col += kPoolThreads) {
      float m = red[0][col];
      for (int r = 1; r < RPP; ++r) m = fmaxf(m, red[r][col]);
      out[DIM + col] = m;
    }
    return;
  }

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;

  uint4 keep[MAXP];
  if (want_r) {
    const T* base = static_cast<const T*>(job.x) + ((size_t)hs * g.n + row0) * DIM + vec * E;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      const int r = rsub + p * RPP;
      keep[p] = (r < nrows) ? ld_stream(base + (size_t)r * DIM) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      float f[E];
      Vec16<T>::to_float(keep[p], f);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] += f[e];
    }
  } else {
    for (int h = 0; h < job.group; ++h) {
      const T* base = static_cast<const T*>(job.x) +
                      ((size_t)(hs * job.group + h) * g.n + row0) * DIM + vec * E;
      int r = rsub;
      for (; r + 3 * RPP < nrows; r += 4 * RPP) {
        uint4 u[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) u[p] = ld_stream(base + (size_t)(r + p * RPP) * DIM);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float f[E];
          Vec16<T>::to_float(u[p], f);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] += f[e];
        }
      }
      for (; r < nrows; r += RPP) {
        float f[E];
        Vec16<T>::to_float(ld_stream(base + (size_t)r * DIM), f);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += f[e];
      }
    }
  }

#pragma unroll
  for (int e = 0; e < E; ++e) red[rsub][vec * E + e] = acc[e];
  __syncthreads();
  const float count = (float)(nrows * job.group);
  for (int col = tid; col < DIM; col += kPoolThreads) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) s += red[r][col];
    const float c = s / count;
    cs[col] = c;
    job.cent[((size_t)hs * g.nb + j) * DIM + col] = c;
  }
  if (!want_r) return;
  __syncthreads();

  float cv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) cv[e] = cs[vec * E + e];
  float best = 0.f;
#pragma unroll
  for (int p = 0; p < MAXP; ++p) {
    const int r = rsub + p * RPP;
    float f[E];
    Vec16<T>::to_float(keep[p], f);
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float dlt = f[e] - cv[e];
      part = fmaf(dlt, dlt, part);
    }
#pragma unroll
    for (int o = VPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (r < nrows) best = fmaxf(best, sqrtf(part));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xFFFFFFFFu, best, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = best;
  __syncthreads();
  if (tid == 0) {
    float m = wmax[0];
#pragma unroll
    for (int w = 1; w < kPoolThreads / 32; ++w) m = fmaxf(m, wmax[w]);
    job.rad[(size_t)hs * g.nb + j] = m;
  }
}

template <typename T, int DIM>
cudaError_t launch_typed(const PoolGrid& g, int total, cudaStream_t s) {
  pool_kernel<T, DIM><<<total, kPoolThreads, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(int dtype, int dim, int seq_len, int block, const PoolJob* jobs, int njobs,
                        cudaStream_t stream) {
  PoolGrid g{};
  g.nb = (seq_len + block - 1) / block;
  g.n = seq_len;
  g.block = block;
  g.job[0] = jobs[0];
  g.job[1] = njobs > 1 ? jobs[1] : jobs[0];
  g.nctas0 = (jobs[0].n_heads / jobs[0].group) * g.nb;
  long long total = g.nctas0;
  if (njobs > 1) total += (long long)(jobs[1].n_heads / jobs[1].group) * g.nb;
  if (total <= 0 || total > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (dtype == SBSA_BF16) {
    return dim == 128 ? launch_typed<__nv_bfloat16, 128>(g, (int)total, stream)
                      : launch_typed<__nv_bfloat16, 64>(g, (int)total, stream);
  }
  return dim == 128 ? launch_typed<float, 128>(g, (int)total, stream)
                    : launch_typed<float, 64>(g, (int)total, stream);
}

}  // namespace sbsa
