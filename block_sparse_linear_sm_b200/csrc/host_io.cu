// The layer on host buffers: copies in, per-unit sla_forward calls and copies
// out, pipelined over three streams. See include/sla.h for the contract.
//
// A unit is one batch entry and a run of whole KV groups (a KV head and the
// query heads that read it). Every head of the layer is computed independently
// of the others (routing, flash tiles, linear states and aggregation are all
// per head), so running a unit as a layer of its own gives bit-identical rows.
#include <string.h>

#include "sla_internal.h"

namespace sla {

namespace {

bool aligned_to(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Arena carve-up: status word, device q / k / v / out, one workspace per unit.
struct HostPlan {
  sla_config unit;  // the configuration of one unit (B = 1, H / n_chunks heads)
  int n_units;
  size_t q_bytes, kv_bytes, out_bytes;  // whole layer
  size_t q_unit, kv_unit;               // one unit's q (= out) and k (= v) bytes
  size_t off_q, off_k, off_v, off_out, off_ws, ws_unit, total;
};

bool make_host_plan(const sla_config* cfg, int32_t n_chunks, HostPlan* hp) {
  if (sla_validate_config(cfg) != SLA_OK) return false;
  if (n_chunks < 1 || cfg->H_kv % n_chunks != 0) return false;
  memset(hp, 0, sizeof(*hp));
  hp->unit = *cfg;
  hp->unit.B = 1;
  hp->unit.H = cfg->H / n_chunks;
  hp->unit.H_kv = cfg->H_kv / n_chunks;
  if (sla_validate_config(&hp->unit) != SLA_OK) return false;
  hp->ws_unit = align_up(sla_workspace_bytes(&hp->unit), 256);
  if (hp->ws_unit == 0) return false;
  hp->n_units = cfg->B * n_chunks;
  const size_t row = (size_t)cfg->N * cfg->d * 2;  // one head's [N, d] bf16
  hp->q_unit = (size_t)hp->unit.H * row;
  hp->kv_unit = (size_t)hp->unit.H_kv * row;
  hp->q_bytes = (size_t)cfg->B * cfg->H * row;
  hp->kv_bytes = (size_t)cfg->B * cfg->H_kv * row;
  hp->out_bytes = hp->q_bytes;
  size_t off = 256;  // status word (two int32) at offset 0
  hp->off_q = off;
  off = align_up(off + hp->q_bytes, 256);
  hp->off_k = off;
  off = align_up(off + hp->kv_bytes, 256);
  hp->off_v = off;
  off = align_up(off + hp->kv_bytes, 256);
  hp->off_out = off;
  off = align_up(off + hp->out_bytes, 256);
  hp->off_ws = off;
  hp->total = off + (size_t)hp->n_units * hp->ws_unit;
  return true;
}

// The first non-zero unit status word (in unit order) goes to the arena's status word.
__global__ void merge_status_kernel(const char* __restrict__ ws0, size_t ws_stride, int n_units,
                                    int* __restrict__ dst) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  for (int u = 0; u < n_units; ++u) {
    const int* st = reinterpret_cast<const int*>(ws0 + (size_t)u * ws_stride);
    if (st[0] != 0) {
      dst[0] = st[0];
      dst[1] = st[1];
      return;
    }
  }
}

}  // namespace

}  // namespace sla

using namespace sla;

extern "C" {

size_t sla_forward_host_device_bytes(const sla_config* cfg, int32_t n_chunks) {
  HostPlan hp;
  return make_host_plan(cfg, n_chunks, &hp) ? hp.total : 0;
}

sla_status sla_forward_host(const void* q_host, const void* k_host, const void* v_host, const void* w_p,
                            const void* w_g, const sla_config* cfg, void* out_host, int32_t n_chunks,
                            void* dev, size_t dev_bytes, void* stream, void* h2d_stream, void* d2h_stream) {
  sla_status st = sla_validate_config(cfg);
  if (st != SLA_OK) return st;
  HostPlan hp;
  if (!make_host_plan(cfg, n_chunks, &hp)) return SLA_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !out_host) return SLA_ERR_INVALID_ARG;
  if (!aligned_to(q_host, 16) || !aligned_to(k_host, 16) || !aligned_to(v_host, 16) || !aligned_to(out_host, 16))
    return SLA_ERR_INVALID_ARG;
  const bool threeway = cfg->mode == SLA_MODE_THREEWAY;
  if (threeway && cfg->has_proj && (!w_p || !aligned_to(w_p, 16))) return SLA_ERR_INVALID_ARG;
  if (cfg->has_gate && (!w_g || !aligned_to(w_g, 16))) return SLA_ERR_INVALID_ARG;
  if (!dev || !aligned_to(dev, 256) || dev_bytes < hp.total) return SLA_ERR_WORKSPACE;

  cudaStream_t s = (cudaStream_t)stream, sin = (cudaStream_t)h2d_stream, sout = (cudaStream_t)d2h_stream;
  char* base = (char*)dev;
  const int n = hp.n_units;
  const int d = cfg->d;
  const size_t wp_head = (size_t)d * d * 2;                               // per-head w_p bytes
  const size_t wg_head = (size_t)(cfg->nsa_branches ? 3 : 1) * d * 2;     // per-head w_g bytes

  // events: start, one per unit arrived, one per unit done, last copy out
  const int n_ev = 2 * n + 2;
  cudaEvent_t ev_small[66];
  cudaEvent_t* ev = n_ev <= 66 ? ev_small : new cudaEvent_t[n_ev];
  int made = 0;
  sla_status result = SLA_OK;
  for (; made < n_ev; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) {
      result = SLA_ERR_CUDA;
      break;
    }
  cudaEvent_t ev_start = ev[0], ev_last = ev[1];
  cudaEvent_t* ev_in = ev + 2;
  cudaEvent_t* ev_done = ev + 2 + n;

  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && result == SLA_OK) result = SLA_ERR_CUDA;
    return result == SLA_OK;
  };
  if (result == SLA_OK) {
    // the arena's status word, then the copies in after everything queued on `stream`
    ok(cudaMemsetAsync(base, 0, 8, s)) && ok(cudaEventRecord(ev_start, s)) &&
        ok(cudaStreamWaitEvent(sin, ev_start, 0)) && ok(cudaStreamWaitEvent(sout, ev_start, 0));
  }
  const int chunks = n_chunks;
  for (int u = 0; u < n && result == SLA_OK; ++u) {
    const int b = u / chunks, c = u % chunks;
    const size_t oq = ((size_t)b * chunks + c) * hp.q_unit;    // bytes into q / out
    const size_t okv = ((size_t)b * chunks + c) * hp.kv_unit;  // bytes into k / v
    ok(cudaMemcpyAsync(base + hp.off_q + oq, (const char*)q_host + oq, hp.q_unit, cudaMemcpyHostToDevice, sin)) &&
        ok(cudaMemcpyAsync(base + hp.off_k + okv, (const char*)k_host + okv, hp.kv_unit, cudaMemcpyHostToDevice,
                           sin)) &&
        ok(cudaMemcpyAsync(base + hp.off_v + okv, (const char*)v_host + okv, hp.kv_unit, cudaMemcpyHostToDevice,
                           sin)) &&
        ok(cudaEventRecord(ev_in[u], sin));
  }
  for (int u = 0; u < n && result == SLA_OK; ++u) {
    const int b = u / chunks, c = u % chunks;
    const size_t oq = ((size_t)b * chunks + c) * hp.q_unit;
    const size_t okv = ((size_t)b * chunks + c) * hp.kv_unit;
    const int h0 = c * hp.unit.H;  // first query head of the unit
    const char* wpu = (const char*)w_p;
    if (threeway && cfg->has_proj && cfg->proj_per_head) wpu += (size_t)h0 * wp_head;
    const char* wgu = cfg->has_gate ? (const char*)w_g + (size_t)h0 * wg_head : (const char*)w_g;
    if (!ok(cudaStreamWaitEvent(s, ev_in[u], 0))) break;
    const sla_status fs = forward_single_stream(base + hp.off_q + oq, base + hp.off_k + okv, base + hp.off_v + okv,
                                                wpu, wgu, &hp.unit, base + hp.off_out + oq, nullptr,
                                                base + hp.off_ws + (size_t)u * hp.ws_unit, hp.ws_unit, s);
    if (fs != SLA_OK) {
      result = fs;
      break;
    }
    ok(cudaEventRecord(ev_done[u], s)) && ok(cudaStreamWaitEvent(sout, ev_done[u], 0)) &&
        ok(cudaMemcpyAsync((char*)out_host + oq, base + hp.off_out + oq, hp.q_unit, cudaMemcpyDeviceToHost, sout));
  }
  if (result == SLA_OK) {
    merge_status_kernel<<<1, 32, 0, s>>>(base + hp.off_ws, hp.ws_unit, n, reinterpret_cast<int*>(base));
    ok(cudaGetLastError()) && ok(cudaEventRecord(ev_last, sout)) && ok(cudaStreamWaitEvent(s, ev_last, 0));
  }
  // an event still pending in a stream is released once it completes
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  if (ev != ev_small) delete[] ev;
  return result;
}

}  // extern "C"
