// sbsa_prefill_host: the prefill from and to host memory, pipelined over
// chunks of kv heads (see include/sbsa.h).
//
// Every kv head's prefill needs only its own K, V and the query heads that
// read it (the percentile gate aside, which averages margins over every
// head), so one request splits into chunks of kv heads whose host -> device
// copies, prefill and device -> host copy overlap: chunk c + 1 is copied in
// while chunk c computes and chunk c - 1 is copied out.  Two staging sets
// in the caller's workspace alternate between chunks; the copies run on two
// streams of the library's own (one per direction, per device), ordered
// against the caller's stream with events.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "internal.h"

namespace sbsa {
namespace {

constexpr int kMaxDevices = 64;

struct CopyStreams {
  cudaStream_t in = nullptr, out = nullptr;
};

// The two copy streams of the current device, created on first use.
bool copy_streams(CopyStreams* cs) {
  static std::mutex mu;
  static CopyStreams cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  CopyStreams& c = cache[dev];
  if (!c.in) {
    if (cudaStreamCreateWithFlags(&c.in, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaStreamCreateWithFlags(&c.out, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(c.in);
      c.in = nullptr;
      return false;
    }
  }
  *cs = c;
  return true;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// How a request is cut: `per` kv heads per chunk, `chunks` chunks.
struct Plan {
  int per, chunks;
  sbsa_params sub;  // the parameters of a full chunk
  size_t q_bytes, kv_bytes, qi_bytes, ki_bytes, o_bytes;  // per chunk
  size_t set_bytes;       // one staging set (inputs and O)
  size_t prefill_bytes;   // the chunk prefill's workspace
  size_t total;
};

bool make_plan(const sbsa_params* p, Plan* pl) {
  const size_t ws = sbsa_prefill_workspace_bytes(p);
  if (ws == 0) return false;
  const int hkv = p->n_kv_heads, group = p->n_q_heads / p->n_kv_heads;
  // one kv head per chunk, except under the percentile gate (one chunk)
  pl->per = p->gate == SBSA_GATE_PERCENTILE ? hkv : 1;
  pl->chunks = (hkv + pl->per - 1) / pl->per;
  pl->sub = *p;
  pl->sub.n_kv_heads = pl->per;
  pl->sub.n_q_heads = pl->per * group;
  const size_t es = p->dtype == SBSA_BF16 ? 2 : 4;
  const size_t n = (size_t)p->seq_len;
  pl->q_bytes = (size_t)pl->sub.n_q_heads * n * p->head_dim * es;
  pl->kv_bytes = (size_t)pl->per * n * p->head_dim * es;
  pl->qi_bytes = p->index_dim ? (size_t)pl->sub.n_q_heads * n * p->index_dim * es : 0;
  pl->ki_bytes = p->index_dim ? (size_t)pl->per * n * p->index_dim * es : 0;
  pl->o_bytes = pl->q_bytes;
  pl->set_bytes = round_up(pl->q_bytes, 256) + 2 * round_up(pl->kv_bytes, 256) +
                  round_up(pl->qi_bytes, 256) + round_up(pl->ki_bytes, 256) +
                  round_up(pl->o_bytes, 256);
  pl->prefill_bytes = sbsa_prefill_workspace_bytes(&pl->sub);
  if (pl->prefill_bytes == 0) return false;
  pl->total = 2 * pl->set_bytes + round_up(pl->prefill_bytes, 256);
  return true;
}

}  // namespace
}  // namespace sbsa

using namespace sbsa;

extern "C" {

size_t sbsa_prefill_host_workspace_bytes(const sbsa_params* p) {
  Plan pl;
  return make_plan(p, &pl) ? pl.total : 0;
}

int sbsa_prefill_host(const sbsa_params* p, const void* q, const void* k, const void* v,
                      const void* q_idx, const void* k_idx, void* o, void* workspace,
                      size_t ws_bytes, void* stream) {
  const int vrc = validate_params(p);
  if (vrc) return vrc;
  Plan pl;
  if (!make_plan(p, &pl)) return SBSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return SBSA_ERR_INVALID_ARG;
  if (p->index_dim && (!q_idx || !k_idx)) return SBSA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < pl.total)
    return SBSA_ERR_WORKSPACE;
  CopyStreams cs;
  if (!copy_streams(&cs)) return SBSA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // events: the caller's prior work, per staging set: inputs in, prefill
  // done, output out
  cudaEvent_t start, in_ready[2], computed[2], out_done[2];
  cudaEvent_t* all[7] = {&start, &in_ready[0], &in_ready[1], &computed[0], &computed[1],
                         &out_done[0], &out_done[1]};
  int made = 0;
  for (; made < 7; ++made)
    if (cudaEventCreateWithFlags(all[made], cudaEventDisableTiming) != cudaSuccess) break;
  auto release = [&]() {
    for (int e = 0; e < made; ++e) cudaEventDestroy(*all[e]);
  };
  if (made < 7) {
    release();
    return SBSA_ERR_CUDA;
  }

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  unsigned char* prefill_ws = ws + 2 * pl.set_bytes;
  const int group = p->n_q_heads / p->n_kv_heads;
  const size_t es = p->dtype == SBSA_BF16 ? 2 : 4;
  const size_t n = (size_t)p->seq_len;
  // bytes of one kv head's slice (and of its query heads') in each tensor
  const size_t kv_head = n * p->head_dim * es, q_head = kv_head * group;
  const size_t ki_head = p->index_dim ? n * p->index_dim * es : 0, qi_head = ki_head * group;

  int rc = SBSA_OK;
  auto check = [&](cudaError_t e) {
    if (e != cudaSuccess && rc == SBSA_OK) rc = SBSA_ERR_CUDA;
    return rc == SBSA_OK;
  };
  check(cudaEventRecord(start, s));
  check(cudaStreamWaitEvent(cs.in, start, 0));
  check(cudaStreamWaitEvent(cs.out, start, 0));
  for (int c = 0; c < pl.chunks && rc == SBSA_OK; ++c) {
    const int b = c & 1;
    const int g0 = c * pl.per;
    const int heads = (g0 + pl.per <= p->n_kv_heads) ? pl.per : p->n_kv_heads - g0;
    sbsa_params sub = pl.sub;
    sub.n_kv_heads = heads;
    sub.n_q_heads = heads * group;
    unsigned char* set = ws + b * pl.set_bytes;
    unsigned char* dq = set;
    unsigned char* dk = dq + round_up(pl.q_bytes, 256);
    unsigned char* dv = dk + round_up(pl.kv_bytes, 256);
    unsigned char* dqi = dv + round_up(pl.kv_bytes, 256);
    unsigned char* dki = dqi + round_up(pl.qi_bytes, 256);
    unsigned char* dout = dki + round_up(pl.ki_bytes, 256);
    // inputs of chunk c into set b, once chunk c - 2's prefill is done with it
    if (c >= 2) check(cudaStreamWaitEvent(cs.in, computed[b], 0));
    const char* hq = static_cast<const char*>(q) + (size_t)g0 * q_head;
    const char* hk = static_cast<const char*>(k) + (size_t)g0 * kv_head;
    const char* hv = static_cast<const char*>(v) + (size_t)g0 * kv_head;
    check(cudaMemcpyAsync(dq, hq, (size_t)heads * q_head, cudaMemcpyHostToDevice, cs.in));
    check(cudaMemcpyAsync(dk, hk, (size_t)heads * kv_head, cudaMemcpyHostToDevice, cs.in));
    check(cudaMemcpyAsync(dv, hv, (size_t)heads * kv_head, cudaMemcpyHostToDevice, cs.in));
    if (p->index_dim) {
      const char* hqi = static_cast<const char*>(q_idx) + (size_t)g0 * qi_head;
      const char* hki = static_cast<const char*>(k_idx) + (size_t)g0 * ki_head;
      check(cudaMemcpyAsync(dqi, hqi, (size_t)heads * qi_head, cudaMemcpyHostToDevice, cs.in));
      check(cudaMemcpyAsync(dki, hki, (size_t)heads * ki_head, cudaMemcpyHostToDevice, cs.in));
    }
    check(cudaEventRecord(in_ready[b], cs.in));
    // the chunk's prefill on the caller's stream, once its inputs are in and
    // chunk c - 2's output has left set b
    check(cudaStreamWaitEvent(s, in_ready[b], 0));
    if (c >= 2) check(cudaStreamWaitEvent(s, out_done[b], 0));
    if (rc != SBSA_OK) break;
    rc = sbsa_prefill(&sub, dq, dk, dv, p->index_dim ? dqi : nullptr,
                      p->index_dim ? dki : nullptr, dout, prefill_ws, pl.prefill_bytes, nullptr,
                      nullptr, nullptr, s);
    if (rc != SBSA_OK) break;
    check(cudaEventRecord(computed[b], s));
    // its output back to the host
    check(cudaStreamWaitEvent(cs.out, computed[b], 0));
    check(cudaMemcpyAsync(static_cast<char*>(o) + (size_t)g0 * q_head, dout,
                          (size_t)heads * q_head, cudaMemcpyDeviceToHost, cs.out));
    check(cudaEventRecord(out_done[b], cs.out));
  }
  // the caller's stream completes after the last outputs (and copies in
  // flight after a failure) have landed
  for (int b = 0; b < 2 && b < pl.chunks; ++b) {
    cudaStreamWaitEvent(s, out_done[b], 0);
    cudaStreamWaitEvent(s, in_ready[b], 0);
  }
  release();
  return rc;
}

}  // extern "C"
