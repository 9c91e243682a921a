// Centroid block scores on the tensor cores.
//
// "Uncertainty-gated selection for block-sparse attention", technical
// summary, Metodologia step 1, and "RBS-Attention", method paragraph (base
// branch): the score of query tile i against key block j is the dot product
// of the tile's pooled query with the block's centroid, s_ij = qbar_i . c_j
// * scale, for every earlier block j < i.  Over all tiles of a head this is
// the lower triangle of the dense product C Qbar^T -- a contraction, so it
// runs as tcgen05 products:
//   D = C_chunk Qbar_chunk^T   (M = 128 candidates, N = 64 query tiles, K = ds)
// with the candidates in TMEM lanes, so thread t of the epilogue owns
// candidate j0 + t and stores one coalesced row segment per query tile.
//
// The selection ranks these scores and is decided in fp32, so the product
// keeps fp32 accuracy with three tf32 products per pair of operands
// (x = hi + lo, hi = x with its low 13 mantissa bits cleared, lo = x - hi,
// exact in fp32):  x.y ~ hi_x hi_y + hi_x lo_y + lo_x hi_y.  The dropped
// lo_x lo_y term and the tf32 rounding of lo are each below 2^-20 |x y|, the
// size of a few fp32 roundings of the sum.
//
// One CTA of 128 threads per (selection head, 64-tile chunk, 128-candidate
// chunk that has a candidate below some tile of the chunk); thread 0 issues
// the TMA copies and the MMAs over K in 32-wide stages, double-buffered;
// every wait is bounded (2 s), after which the CTA records SBSA_ERR_TIMEOUT
// and leaves once its copies and products have drained.
#include <cuda.h>

#include "internal.h"
#include "ptx.cuh"
#include "tma_map.h"

namespace sbsa {
namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kThreads = 128;
constexpr int kCand = 128;  // candidates per CTA (M, TMEM lanes)
constexpr int kTiles = 64;  // query tiles per CTA (N, TMEM columns)

struct CsParams {
  CUtensorMap tm_ch, tm_cl;  // centroids hi / lo [Hkv, NB, ds], fp32
  CUtensorMap tm_qh, tm_ql;  // pooled queries hi / lo [Hs, NB, ds], fp32
  float* scores;             // [Hs, NB, NB]; row (hs, i) holds candidates j < i
  int nb, kv_div, n_jc;
  float scale;
  int* status;
};

// One K stage: 32 fp32 columns (one 128-byte swizzle atom) of each operand.
constexpr int A_BYTES = kCand * 128;   // 16 KB
constexpr int B_BYTES = kTiles * 128;  // 8 KB
constexpr int OFF_AH = 0;
constexpr int OFF_AL = A_BYTES;
constexpr int OFF_BH = 2 * A_BYTES;
constexpr int OFF_BL = 2 * A_BYTES + B_BYTES;
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;  // 48 KB
constexpr int SMEM_BYTES = 2 * STAGE_BYTES + 1024;      // two stages + alignment slack
constexpr uint32_t IDESC = make_idesc(2, kCand, kTiles, false, false);
constexpr int TM_COLS = 64;

__device__ __forceinline__ void record(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// hi = x with the 13 low mantissa bits cleared (exactly a tf32 value),
// lo = x - hi (exact), for two arrays in one grid (counts in float4s).
__global__ void __launch_bounds__(256) split_tf32_kernel(const float4* __restrict__ x0,
                                                         float4* __restrict__ hi0,
                                                         float4* __restrict__ lo0, size_t n0,
                                                         const float4* __restrict__ x1,
                                                         float4* __restrict__ hi1,
                                                         float4* __restrict__ lo1, size_t n1) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n0 + n1;
       e += (size_t)gridDim.x * blockDim.x) {
    const bool first = e < n0;
    const size_t at = first ? e : e - n0;
    const float4 v = first ? x0[at] : x1[at];
    float4 h;
    h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
    h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
    h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
    h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
    const float4 l = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
    (first ? hi0 : hi1)[at] = h;
    (first ? lo0 : lo1)[at] = l;
  }
}

template <int DS>
__global__ void __launch_bounds__(kThreads) centroid_scores_kernel(const __grid_constant__ CsParams p) {
  constexpr int NS = DS / 32;  // K stages
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  __shared__ uint64_t full[2], empty[2], d_full;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int hs = blockIdx.y;
  const int ic = (int)blockIdx.x / p.n_jc;
  const int jc = (int)blockIdx.x % p.n_jc;
  const int i0 = ic * kTiles;
  const int j0 = jc * kCand;
  // largest query tile of the chunk; candidates j < i_last are needed
  const int i_last = min(i0 + kTiles, p.nb) - 1;
  if (j0 >= i_last) return;  // uniform over the CTA, before any barrier
  const int g = hs / p.kv_div;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&empty[b], 1);
    }
    mbar_init(&d_full, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, TM_COLS);
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

  bool ok = true;
  if (tid == 0) {
    tma_prefetch_desc(&p.tm_ch);
    tma_prefetch_desc(&p.tm_cl);
    tma_prefetch_desc(&p.tm_qh);
    tma_prefetch_desc(&p.tm_ql);
    const uint32_t base = smem_u32(smem);
    auto load = [&](int s) {
      unsigned char* st = smem + (s & 1) * STAGE_BYTES;
      mbar_arrive_expect_tx(&full[s & 1], STAGE_BYTES);
      tma_load_3d(st + OFF_AH, &p.tm_ch, &full[s & 1], s * 32, j0, g);
      tma_load_3d(st + OFF_AL, &p.tm_cl, &full[s & 1], s * 32, j0, g);
      tma_load_3d(st + OFF_BH, &p.tm_qh, &full[s & 1], s * 32, i0, hs);
      tma_load_3d(st + OFF_BL, &p.tm_ql, &full[s & 1], s * 32, i0, hs);
    };
    int loaded = 0, issued = 0;
    for (; loaded < 2 && loaded < NS; ++loaded) load(loaded);
    for (int s = 0; s < NS && ok; ++s) {
      ok = wait(&full[s & 1], (s >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint32_t st = base + (s & 1) * STAGE_BYTES;
      const uint64_t ah = smem_desc(st + OFF_AH, 16, 1024);
      const uint64_t al = smem_desc(st + OFF_AL, 16, 1024);
      const uint64_t bh = smem_desc(st + OFF_BH, 16, 1024);
      const uint64_t bl = smem_desc(st + OFF_BL, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // 8 tf32 (32 bytes) per instruction
        const uint64_t off = (uint64_t)((kk * 32) >> 4);
        umma_tf32_ss(tmem, al + off, bh + off, IDESC, (s > 0 || kk > 0) ? 1u : 0u);
        umma_tf32_ss(tmem, ah + off, bl + off, IDESC, 1u);
        umma_tf32_ss(tmem, ah + off, bh + off, IDESC, 1u);
      }
      umma_commit(&empty[s & 1]);
      ++issued;
      if (loaded < NS) {
        // the buffer is reused once the products that read it are done
        ok = wait(&empty[s & 1], (s >> 1) & 1);
        if (ok) load(loaded++);
      }
    }
    if (ok) {
      umma_commit(&d_full);
    } else {
      if (!abort_flag) {
        abort_flag = 1;
        record(p.status, SBSA_ERR_TIMEOUT);
      }
      // copies still in flight land in this CTA's shared memory, and
      // products still running read it: let both finish before leaving
      volatile int never = 0;
      for (int s = issued; s < loaded; ++s)
        mbar_wait_bounded(&full[s & 1], (s >> 1) & 1, &never, kTimeoutNs);
      if (issued > 0) {
        umma_commit(&d_full);
        mbar_wait_bounded(&d_full, 0, &never, kTimeoutNs);
      }
    }
  }
  ok = wait(&d_full, 0) && !abort_flag;
  if (__syncthreads_and(ok)) {
    tc_fence_after();
    const int j = j0 + tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll
    for (int c0 = 0; c0 < kTiles; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int i = i0 + c0 + c;
        if (i < p.nb && j < i) p.scores[((size_t)hs * p.nb + i) * p.nb + j] = v[c] * p.scale;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

template <int DS>
cudaError_t launch_ds(const CentroidScoreArgs& a, cudaStream_t stream) {
  CsParams p{};
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!make_map(&p.tm_ch, dt, 4, a.c_hi, a.hkv, a.nb, DS, kCand) ||
      !make_map(&p.tm_cl, dt, 4, a.c_lo, a.hkv, a.nb, DS, kCand) ||
      !make_map(&p.tm_qh, dt, 4, a.q_hi, a.hs, a.nb, DS, kTiles) ||
      !make_map(&p.tm_ql, dt, 4, a.q_lo, a.hs, a.nb, DS, kTiles))
    return cudaErrorInvalidValue;
  p.scores = a.scores;
  p.nb = a.nb;
  p.kv_div = a.kv_div;
  p.n_jc = (a.nb + kCand - 1) / kCand;
  p.scale = a.scale;
  p.status = a.status;
  auto kern = centroid_scores_kernel<DS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  if (a.nb < 2) return cudaSuccess;  // no tile has candidates
  const long long n_ic = (a.nb + kTiles - 1) / kTiles;
  const long long gx = n_ic * p.n_jc;
  if (gx > 0x7FFFFFFFLL || a.hs > 65535) return cudaErrorInvalidValue;
  kern<<<dim3((unsigned)gx, a.hs), kThreads, SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_centroid_scores(const CentroidScoreArgs& a, cudaStream_t stream) {
  const size_t nq = (size_t)a.hs * a.nb * a.ds / 4, nk = (size_t)a.hkv * a.nb * a.ds / 4;
  const size_t want = (nq + nk + 255) / 256;
  const int blocks = (int)(want < 4096 ? want : 4096);
  split_tf32_kernel<<<blocks, 256, 0, stream>>>(
      reinterpret_cast<const float4*>(a.qc), reinterpret_cast<float4*>(a.q_hi),
      reinterpret_cast<float4*>(a.q_lo), nq, reinterpret_cast<const float4*>(a.kc),
      reinterpret_cast<float4*>(a.c_hi), reinterpret_cast<float4*>(a.c_lo), nk);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return a.ds == 128 ? launch_ds<128>(a, stream) : launch_ds<64>(a, stream);
}

}  // namespace sbsa
