// Row-max tile scores on the tensor cores.
//
// "Uncertainty-gated selection for block-sparse attention", technical
// summary, Metodologia step 2: selection runs per query tile, and a tile's
// score for a key block is the largest score among the tile's query rows.
// With the mean-pooling backbone a row's score is q_t . c_j, so the tile
// score s_ij = max_t q_t . c_j * scale is a dense contraction followed by a
// maximum -- tcgen05 products per (tile, chunk of 128 candidate blocks):
//   D = C_chunk Q_tile^T   (M = 128 candidates, N = 128 query rows, K = d)
// with the candidates in TMEM lanes, so each thread reduces its own lane
// (one candidate) over the tile's valid query rows.  In group mode the rows
// of every head of the group are maximised over as well.
//
// Precision: the page's score is the plain dot product with the fp32
// centroids.  A conversion kernel splits every centroid into three bf16
// parts, c = c_hi + c_mid + c_lo (c_hi = bf16(c), c_mid = bf16(c - c_hi),
// c_lo = bf16(c - c_hi - c_mid), round to nearest even).  The 24-bit fp32
// significand fits in the three 8-bit ones, so the split is exact for every
// centroid of magnitude above 2^-100; the query rows are bf16, so each
// product q * c_part is exact in fp32 too.  D accumulates the three products
// (smallest part first) in fp32: the only rounding is the tensor core's
// accumulation.
//
// One CTA of 128 threads per (selection head, query tile i >= 1): thread 0
// issues the TMA copies and the MMAs; the centroid part tiles stream through
// a 4-stage ring, D is double-buffered; every wait is bounded (2 s), after
// which the CTA records SBSA_ERR_TIMEOUT and leaves once its copies and
// products have drained.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tma_map.h"

namespace sbsa {

namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kThreads = 128;
constexpr int kStages = 4;  // centroid part tiles in flight
constexpr int kParts = 3;   // bf16 parts per centroid

struct RowmaxParams {
  CUtensorMap tm_q;  // Q (or Q_idx) [Hq, N, ds], bf16
  CUtensorMap tm_c;  // centroid parts [3 * Hkv, NB, ds], bf16 (part p of kv head g at p * Hkv + g)
  float* scores;     // [Hs, NB, NB]; row (hs, i) holds candidates j < i
  int n, nb, hkv, group, group_shared;
  float scale;
  int* status;
};

template <int DS>
struct RM {
  static constexpr int NA = DS / 64;                          // 128-byte swizzle atoms across ds
  static constexpr int TILE_BYTES = 128 * DS * 2;             // 128 rows of ds bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_C = TILE_BYTES;                    // ring[kStages]
  static constexpr int OFF_MAX = (1 + kStages) * TILE_BYTES;  // running maxima [chunks][128]
  static constexpr uint32_t IDESC = make_idesc(1, 128, 128, false, false);
};

__device__ __forceinline__ void record(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// The exact three-part bf16 split of each fp32 centroid, into three planes
// of [Hkv, NB, ds] (hi, mid, lo).
__global__ void __launch_bounds__(256) split3_kernel(const float* __restrict__ x,
                                                     __nv_bfloat16* __restrict__ parts, size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const float c = x[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(c);
    const float r1 = c - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    parts[e] = hi;
    parts[n + e] = mid;
    parts[2 * n + e] = __float2bfloat16_rn(r2);
  }
}

template <int DS>
__global__ void __launch_bounds__(kThreads) rowmax_kernel(const __grid_constant__ RowmaxParams p) {
  using C = RM<DS>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  __shared__ uint64_t q_full, c_full[kStages], c_free[kStages], d_full[2], d_free[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int hs = blockIdx.y;
  const int i = blockIdx.x + 1;  // query tile; tile 0 has no candidates
  const int nrows = min(128, p.n - i * 128);
  const int nchunks = (i + 127) / 128;
  const int heads = p.group_shared ? p.group : 1;
  const int h0 = p.group_shared ? hs * p.group : hs;  // first query head of the tile
  const int g = p.group_shared ? hs : hs / p.group;   // kv head of the centroids
  float* run_max = reinterpret_cast<float*>(smem + C::OFF_MAX);

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&drain, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_free[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&d_full[b], 1);
      mbar_init(&d_free[b], kThreads);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  for (int e = tid; e < nchunks * 128; e += kThreads) run_max[e] = -INFINITY;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;
  auto wait = [&](uint64_t* b, uint32_t parity) {
    return mbar_wait_bounded(b, parity, abort_v, kTimeoutNs);
  };

  // step s: head s / nchunks, chunk s % nchunks; load l: step l / 3, part
  // 2 - l % 3 (lo, mid, hi: the smallest parts are accumulated first)
  const int steps = heads * nchunks;
  const int loads = steps * kParts;
  const uint32_t q_base = smem_u32(smem + C::OFF_Q);
  const uint32_t c_base = smem_u32(smem + C::OFF_C);
  auto load_c = [&](int l) {
    const int st = l % kStages;
    const int s = l / kParts;
    const int part = kParts - 1 - l % kParts;
    mbar_arrive_expect_tx(&c_full[st], C::TILE_BYTES);
    for (int a = 0; a < C::NA; ++a)
      tma_load_3d(smem + C::OFF_C + st * C::TILE_BYTES + a * (128 * 128), &p.tm_c, &c_full[st],
                  a * 64, (s % nchunks) * 128, part * p.hkv + g);
  };
  bool ok = true;
  int issued = 0;    // MMA chains issued (thread 0)
  int loaded = 0;    // part tiles requested (thread 0)
  int consumed = 0;  // part tiles multiplied (thread 0)
  int drains = 0;    // commits to `drain` so far (thread 0)
  if (tid == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_c);
    for (; loaded < kStages - 1 && loaded < loads; ++loaded) load_c(loaded);
  }
  for (int s = 0; s <= steps && ok; ++s) {
    if (tid == 0 && s < steps) {
      const int chunk = s % nchunks;
      const int h = s / nchunks;
      if (chunk == 0) {
        // Q of head h: the previous head's products must be done with it
        if (h > 0) {
          umma_commit(&drain);
          ok = wait(&drain, drains & 1);
          ++drains;
        }
        if (ok) {
          mbar_arrive_expect_tx(&q_full, C::TILE_BYTES);
          for (int a = 0; a < C::NA; ++a)
            tma_load_3d(smem + C::OFF_Q + a * (128 * 128), &p.tm_q, &q_full, a * 64, i * 128,
                        h0 + h);
          ok = wait(&q_full, h & 1);
        }
      }
      // D[s % 2] is free once every thread has read step s - 2
      if (ok && s >= 2) ok = wait(&d_free[s & 1], ((s - 2) >> 1) & 1);
      for (int pp = 0; pp < kParts && ok; ++pp) {
        const int l = s * kParts + pp;
        const int st = l % kStages;
        ok = wait(&c_full[st], (l / kStages) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad0 = smem_desc(c_base + st * C::TILE_BYTES, 16, 1024);
        const uint64_t bd0 = smem_desc(q_base, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < DS / 16; ++kk) {
          const int kb = kk * 32;
          const uint64_t off = (uint64_t)(((kb / 128) * (128 * 128) + (kb % 128)) >> 4);
          umma_f16_ss(tmem + (s & 1) * 128, ad0 + off, bd0 + off, C::IDESC,
                      (pp > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&c_free[st]);
        ++issued;
        ++consumed;
        if (pp == kParts - 1) umma_commit(&d_full[s & 1]);
        // refill the stage of the previous part tile once its product is done
        if (loaded < loads) {
          if (loaded >= kStages) ok = wait(&c_free[loaded % kStages], ((loaded - kStages) / kStages) & 1);
          if (ok) load_c(loaded++);
        }
      }
      if (!ok && !abort_flag) {
        abort_flag = 1;
        record(p.status, SBSA_ERR_TIMEOUT);
      }
    }
    // every thread: reduce step s - 1 (its own candidate, over the valid rows)
    if (s >= 1) {
      const int r = s - 1;
      if (!wait(&d_full[r & 1], (r >> 1) & 1)) ok = false;
      if (!__syncthreads_and(ok)) break;
      tc_fence_after();
      const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
      float m = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + (r & 1) * 128 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c0 + c < nrows) m = fmaxf(m, v[c]);
      }
      tc_fence_before();
      mbar_arrive(&d_free[r & 1]);
      float* slot = run_max + (r % nchunks) * 128 + tid;
      *slot = fmaxf(*slot, m);
    }
    if (!__syncthreads_and(ok && !abort_flag)) {
      ok = false;
      break;
    }
  }
  if (ok) {
    // candidate j = chunk * 128 + tid of tile i, for j < i
    float* out = p.scores + ((size_t)hs * p.nb + i) * p.nb;
    for (int chunk = 0; chunk < nchunks; ++chunk) {
      const int j = chunk * 128 + tid;
      if (j < i) out[j] = run_max[chunk * 128 + tid] * p.scale;
    }
  } else if (tid == 0) {
    // let the products already issued finish before TMEM is released, and
    // the part tiles still in flight land in this CTA's shared memory
    volatile int never = 0;
    if (issued > 0) {
      umma_commit(&drain);
      mbar_wait_bounded(&drain, drains & 1, &never, kTimeoutNs);
    }
    for (int l = consumed; l < loaded; ++l)
      mbar_wait_bounded(&c_full[l % kStages], (l / kStages) & 1, &never, kTimeoutNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int DS>
size_t smem_bytes(int nb) {
  const int nchunks_max = (nb - 1 + 127) / 128;
  return (size_t)(1 + kStages) * RM<DS>::TILE_BYTES + (size_t)nchunks_max * 128 * 4 + 1024;
}

template <int DS>
cudaError_t launch_ds(const RowmaxArgs& a, cudaStream_t stream) {
  RowmaxParams p{};
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&p.tm_q, dt, 2, a.q, a.hq, a.n, DS, 128) ||
      !make_map(&p.tm_c, dt, 2, a.c_parts, 3 * a.hkv, a.nb, DS, 128))
    return cudaErrorInvalidValue;
  p.scores = a.scores;
  p.n = a.n;
  p.nb = a.nb;
  p.hkv = a.hkv;
  p.group = a.hq / a.hkv;
  p.group_shared = a.group_shared;
  p.scale = a.scale;
  p.status = a.status;
  const size_t smem = smem_bytes<DS>(a.nb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = rowmax_kernel<DS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  const int hs = a.group_shared ? a.hkv : a.hq;
  if (a.nb < 2) return cudaSuccess;  // no tile has candidates
  dim3 grid(a.nb - 1, hs);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool rowmax_fits(int nb, int ds) {
  return (ds == 128 ? smem_bytes<128>(nb) : smem_bytes<64>(nb)) <= 227 * 1024;
}

cudaError_t launch_rowmax(const RowmaxArgs& a, cudaStream_t stream) {
  const size_t n = (size_t)a.hkv * a.nb * a.ds;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  split3_kernel<<<blocks, 256, 0, stream>>>(a.c_f32, a.c_parts, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return a.ds == 128 ? launch_ds<128>(a, stream) : launch_ds<64>(a, stream);
}

}  // namespace sbsa
