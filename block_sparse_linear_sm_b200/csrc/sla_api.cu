// C ABI of the sparse+linear attention layer: validation, workspace plan and
// the launch sequence. See include/sla.h for the contract of each entry point.
#include <mutex>
#include <math.h>
#include <string.h>

#include "sla_internal.h"

namespace sla {

static sla_status check_config(const sla_config* c) {
  if (c == nullptr) return SLA_ERR_INVALID_ARG;
  if (c->B < 1 || c->H < 1 || c->H_kv < 1 || c->N < 1 || c->d < 1 || c->block < 1)
    return SLA_ERR_INVALID_ARG;
  if (c->H % c->H_kv != 0) return SLA_ERR_INVALID_ARG;
  if (c->N % c->block != 0) return SLA_ERR_INVALID_ARG;
  if (c->N_valid > c->N || c->N_valid <= c->N - c->block) return SLA_ERR_INVALID_ARG;
  if (!(c->scale >= 0.f) || !isfinite(c->scale)) return SLA_ERR_INVALID_ARG;
  if ((c->cos_filter != 0 && c->cos_filter != 1) || !isfinite(c->cos_theta)) return SLA_ERR_INVALID_ARG;
  if (c->block != kBlock) return SLA_ERR_UNSUPPORTED;
  if (c->d != 64 && c->d != 128) return SLA_ERR_UNSUPPORTED;
  const int nb = c->N / c->block;
  if (nb > kMaxBlocks) return SLA_ERR_UNSUPPORTED;
  if ((int64_t)c->B * c->H * c->N * c->d > ((int64_t)1 << 40)) return SLA_ERR_UNSUPPORTED;
  if (c->nsa_branches != 0 && c->nsa_branches != 1) return SLA_ERR_INVALID_ARG;
  if (c->mode == SLA_MODE_THREEWAY) {
    if (c->k_h < 0 || c->k_l < 0 || c->k_h + c->k_l > nb) return SLA_ERR_INVALID_ARG;
    if (c->nsa_branches != 0) return SLA_ERR_UNSUPPORTED;
    if (c->causal != 0) return SLA_ERR_UNSUPPORTED;
    if ((c->has_proj != 0 && c->has_proj != 1) || (c->has_gate != 0 && c->has_gate != 1) ||
        (c->proj_per_head != 0 && c->proj_per_head != 1) || (c->smooth_k != 0 && c->smooth_k != 1) ||
        (c->linear_all != 0 && c->linear_all != 1))
      return SLA_ERR_INVALID_ARG;
    if (c->proj_per_head && (!c->has_proj || c->H_kv != c->H)) return SLA_ERR_UNSUPPORTED;
  } else if (c->mode == SLA_MODE_TOPN_WINDOW) {
    if (c->top_n < 0 || c->window < 0) return SLA_ERR_INVALID_ARG;
    if (c->causal != 1) return SLA_ERR_UNSUPPORTED;
    if (c->has_proj != 0 || c->proj_per_head != 0 || c->smooth_k != 0 || c->linear_all != 0)
      return SLA_ERR_UNSUPPORTED;
    if (c->has_gate != 0 && c->has_gate != 1) return SLA_ERR_INVALID_ARG;
    if (c->has_gate && !c->nsa_branches) return SLA_ERR_UNSUPPORTED;  // gates belong to NSA's branches
    if (c->nsa_branches) {
      if (c->cmp_block < 1 || c->cmp_stride < 1) return SLA_ERR_INVALID_ARG;
      if (c->cmp_block > 1024 || c->cmp_stride > 1024) return SLA_ERR_UNSUPPORTED;
    }
    // selected blocks plus window blocks must fit the kernel's 128-entry list
    if (c->top_n > 64 || c->top_n + (c->window + 62) / kBlock + 1 > 128) return SLA_ERR_UNSUPPORTED;
  } else {
    return SLA_ERR_INVALID_ARG;
  }
  return SLA_OK;
}

bool make_plan(const sla_config* c, Plan* p) {
  if (check_config(c) != SLA_OK) return false;
  memset(p, 0, sizeof(*p));
  p->c = *c;
  p->nqb = p->nkb = c->N / kBlock;
  p->group = c->H / c->H_kv;
  p->nqb_pad = (int)align_up(p->nqb, 128);
  p->nkb_pad = (int)align_up(p->nkb, 64);
  p->qb0 = 0;
  p->qb1 = p->nqb;
  p->dd = (int)align_up((size_t)c->d * c->d + c->d, 128);
  p->scale = c->scale > 0.f ? c->scale : 1.f / sqrtf((float)c->d);
  const size_t B = c->B, H = c->H, Hkv = c->H_kv, d = c->d, nqb = p->nqb, nkb = p->nkb;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  p->off_status = take(256);
  p->off_qbar = take(B * H * nqb * d * 8);
  p->off_kbar = take(B * Hkv * nkb * d * 8);
  p->off_scores = take(B * H * nqb * nkb * 8);
  if (c->cos_filter) p->off_kflag = take(B * Hkv * nkb);  // 1: the key block's pooled scores are -inf
  if (c->mode == SLA_MODE_THREEWAY) {
    p->off_crit = take(B * H * nqb * (size_t)c->k_h * 4);
    p->off_neg = off;
    p->off_lse = take(B * H * (size_t)c->N * 4);  // row log2-sum-exp of the sparse branch (backward)
    const bool marginal = p->nkb - c->k_h - c->k_l > 0 || c->linear_all;
    if (marginal) {
      p->off_mmask = take(B * H * (size_t)p->nqb_pad * p->nkb_pad * 2);
      p->off_hs = take(B * Hkv * (size_t)p->nkb_pad * p->dd * 2);
      p->off_ss = take(B * H * nqb * d * d * 2);  // S_i (times W_p), bf16
      p->off_zs = take(B * H * nqb * d * 4);      // Z_i, fp32
      p->off_phiq = take(B * H * (size_t)c->N * d * 2);  // phi(Q), bf16
      if (c->has_gate) p->off_gate = take(B * H * (size_t)c->N * 4);  // sigmoid(q . w_g), fp32
      if (c->smooth_k) p->off_kmean = take(B * Hkv * d * 4);            // mean valid key, fp32
    }
  } else {
    p->off_crit = take(B * Hkv * nqb * (size_t)c->top_n * 4);
    // row log2-sum-exp of the sparse branch (backward); NSA: one row per branch
    p->off_lse = take((c->nsa_branches ? 3 : 1) * B * H * (size_t)c->N * 4);
    if (c->nsa_branches) {
      // compressed blocks that hold valid tokens only, padded to whole 64-key tiles
      p->n_cmp = c->N_valid >= c->cmp_block ? (c->N_valid - c->cmp_block) / c->cmp_stride + 1 : 0;
      p->ncmp_pad = (int)align_up((size_t)(p->n_cmp > 0 ? p->n_cmp : 1), 64);
      p->off_kc = take(B * Hkv * (size_t)p->ncmp_pad * d * 2);
      p->off_vc = take(B * Hkv * (size_t)p->ncmp_pad * d * 2);
      p->off_oc = take(B * H * (size_t)c->N * d * 2);
      p->off_os = take(B * H * (size_t)c->N * d * 2);
      p->off_ow = take(B * H * (size_t)c->N * d * 2);  // window branch output (backward)
    }
  }
  p->total = off;
  return true;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static bool has_marginal(const Plan& p) { return p.nkb - p.c.k_h - p.c.k_l > 0 || p.c.linear_all; }

// Stage list of a configuration.
enum Stage { kPool, kScores, kClassify, kSelect, kState, kAggregate, kFlash, kCompress, kFlashCmp, kFlashSlc,
             kFlashWin };
constexpr int kMaxStages = 12;

static int stages_of(const Plan& p, Stage* out) {
  int n = 0;
  out[n++] = kPool;
  out[n++] = kScores;
  if (p.c.mode == SLA_MODE_THREEWAY) {
    out[n++] = kClassify;
    if (has_marginal(p)) {
      out[n++] = kState;
      out[n++] = kAggregate;
    }
    out[n++] = kFlash;  // with a linear branch its tail runs the layer's epilogue
  } else {
    out[n++] = kSelect;
    if (p.c.nsa_branches) {  // NSA's three branches; the last one sums them with their gates
      out[n++] = kCompress;
      out[n++] = kFlashCmp;
      out[n++] = kFlashSlc;
      out[n++] = kFlashWin;  // its epilogue writes the gated sum of the three branches
    } else {
      out[n++] = kFlash;
    }
  }
  return n;
}

static const char* stage_name(Stage s) {
  switch (s) {
    case kPool: return "pool";
    case kScores: return "pooled_scores";
    case kClassify: return "classify";
    case kSelect: return "select_topn";
    case kState: return "linear_state";
    case kAggregate: return "linear_aggregate";
    case kFlash: return "sparse_flash";
    case kCompress: return "compress_kv";
    case kFlashCmp: return "sparse_flash_cmp";
    case kFlashSlc: return "sparse_flash_slc";
    case kFlashWin: return "sparse_flash_win";
  }
  return "?";
}

static cudaError_t run_stage(Stage st, const Plan& p, const Args& a, cudaStream_t s) {
  switch (st) {
    case kPool: return launch_pool(p, a, s);
    case kScores: return launch_scores(p, a, s);
    case kClassify: return launch_classify(p, a, /*write_mmask=*/has_marginal(p), s);
    case kSelect: return launch_select(p, a, s);
    case kState: return launch_state(p, a, s);
    case kAggregate: return launch_aggregate(p, a, s);
    case kFlash: return launch_flash(p, a, s);
    case kCompress: return launch_compress(p, a, s);
    case kFlashCmp: return launch_flash_nsa(p, a, 1, s);
    case kFlashSlc: return launch_flash_nsa(p, a, 2, s);
    case kFlashWin: return launch_flash_nsa(p, a, 3, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t route_stages(const Plan& p, const Args& a, cudaStream_t s) {
  cudaError_t e = launch_pool(p, a, s);
  if (e == cudaSuccess) e = launch_scores(p, a, s);
  if (e == cudaSuccess) e = p.c.mode == SLA_MODE_THREEWAY ? launch_classify(p, a, false, s) : launch_select(p, a, s);
  return e;
}

// The library's side stream of the current device and context (created on first use,
// non-blocking, kept until the process exits), or null when the context cannot be told
// apart. The linear-state stage runs on it beside the routing.
static cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  static unsigned long long ctxs[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (streams[dev] == nullptr || ctxs[dev] != ctx) {
    cudaStream_t st = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    streams[dev] = st;
    ctxs[dev] = ctx;
  }
  return streams[dev];
}

static sla_status forward_impl(const void* q, const void* k, const void* v, const void* w_p,
                               const void* w_g, const sla_config* cfg, void* out, int8_t* mask_out,
                               void* ws, size_t ws_bytes, void* stream, void* const* events,
                               int32_t n_events, int32_t qb_begin = 0, int32_t qb_end = -1,
                               bool may_fork = true) {
  Plan p;
  sla_status st = check_config(cfg);
  if (st != SLA_OK) return st;
  make_plan(cfg, &p);
  if (qb_end < 0) qb_end = p.nqb;
  // a range of query blocks starts on a pair of blocks (the flash kernel's 128-row units)
  if (qb_begin < 0 || qb_begin >= qb_end || qb_end > p.nqb || (qb_begin & 1) || ((qb_end & 1) && qb_end != p.nqb))
    return SLA_ERR_INVALID_ARG;
  p.qb0 = qb_begin;
  p.qb1 = qb_end;
  if (!q || !k || !v || !out) return SLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return SLA_ERR_INVALID_ARG;
  const bool threeway = cfg->mode == SLA_MODE_THREEWAY;
  if (threeway && cfg->has_proj && (!w_p || !aligned(w_p, 16))) return SLA_ERR_INVALID_ARG;
  if (cfg->has_gate && (!w_g || !aligned(w_g, 16))) return SLA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return SLA_ERR_WORKSPACE;
  Stage stages[kMaxStages];
  const int ns = stages_of(p, stages);
  if (events && n_events != ns + 1) return SLA_ERR_INVALID_ARG;

  Args a;
  memset(&a, 0, sizeof(a));
  a.q = (const __nv_bfloat16*)q;
  a.k = (const __nv_bfloat16*)k;
  a.v = (const __nv_bfloat16*)v;
  a.w_p = (const __nv_bfloat16*)w_p;
  a.w_g = (const __nv_bfloat16*)w_g;
  a.out = (__nv_bfloat16*)out;
  a.mask_out = mask_out;
  a.ws = (char*)ws;
  a.status = (int*)((char*)ws + p.off_status);
  a.crit = (int32_t*)((char*)ws + p.off_crit);
  a.neg = nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(a.status, 0, 8, s) != cudaSuccess) return SLA_ERR_CUDA;
  // The linear states need only K and V (and, with smooth-K, the pooled keys): after the
  // pooling pass they run on the side stream while the pooled scores and the
  // classification run on `stream`, which waits for them before the aggregation. A call
  // that times its stages runs them in order on `stream`.
  cudaStream_t side = (may_fork && !events) ? side_stream() : nullptr;
  bool has_state = false;
  for (int i = 0; i < ns; ++i) has_state = has_state || stages[i] == kState;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  if (side && has_state) {
    if (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess) return SLA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess) {
      cudaEventDestroy(ev_fork);
      return SLA_ERR_CUDA;
    }
  } else {
    side = nullptr;
  }
  sla_status result = SLA_OK;
  if (events && cudaEventRecord((cudaEvent_t)events[0], s) != cudaSuccess) result = SLA_ERR_CUDA;
  for (int i = 0; i < ns && result == SLA_OK; ++i) {
    if (side && stages[i] == kState) continue;  // already enqueued on the side stream
    if (side && stages[i] == kAggregate && cudaStreamWaitEvent(s, ev_join, 0) != cudaSuccess) {
      result = SLA_ERR_CUDA;
      break;
    }
    if (run_stage(stages[i], p, a, s) != cudaSuccess) {
      result = SLA_ERR_CUDA;
      break;
    }
    if (side && stages[i] == kPool &&
        (cudaEventRecord(ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess ||
         run_stage(kState, p, a, side) != cudaSuccess || cudaEventRecord(ev_join, side) != cudaSuccess)) {
      result = SLA_ERR_CUDA;
      break;
    }
    if (events && cudaEventRecord((cudaEvent_t)events[i + 1], s) != cudaSuccess) result = SLA_ERR_CUDA;
  }
  if (side) {
    // the events are released once they have completed
    cudaEventDestroy(ev_fork);
    cudaEventDestroy(ev_join);
  }
  return result;
}

sla_status forward_single_stream(const void* q, const void* k, const void* v, const void* w_p, const void* w_g,
                                 const sla_config* cfg, void* out, int8_t* mask_out, void* ws, size_t ws_bytes,
                                 void* stream) {
  return forward_impl(q, k, v, w_p, w_g, cfg, out, mask_out, ws, ws_bytes, stream, nullptr, 0, 0, -1, false);
}

// ---------------------------------------------------------------------------
// backward pass
// ---------------------------------------------------------------------------
static sla_status check_bwd_config(const sla_config* c) { return check_config(c); }

bool make_bwd_plan(const Plan& p, BwdPlan* b) {
  memset(b, 0, sizeof(*b));
  const sla_config& c = p.c;
  b->lin = c.mode == SLA_MODE_THREEWAY && has_marginal(p);  // the top-n mode has no linear branch
  b->nsa = c.mode == SLA_MODE_TOPN_WINDOW && c.nsa_branches;
  b->rows_t = p.group * p.nqb_pad;
  b->words = (p.nqb + 31) / 32;
  const size_t B = c.B, H = c.H, Hkv = c.H_kv, d = c.d, N = c.N;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  b->off_status = take(256);
  b->off_ctr = take(256);
  b->off_delta = take((b->nsa ? 3 : 1) * B * H * N * 4);     // D_t = dO_t . O_s,t (NSA: dO_t . o_b,t)
  b->off_bits = take(B * H * p.nkb * (size_t)b->words * 4);  // query blocks of each key block
  // merged (query head, query block) list of each pair of key blocks
  b->off_dlist = take(B * Hkv * (size_t)((p.nkb + 1) / 2) * dkdv_list_cap(p) * 4);
  if (c.mode == SLA_MODE_TOPN_WINDOW)
    b->off_lbits = take(B * Hkv * (size_t)((p.nkb + 1) / 2) * 4 * b->words * 4);
  if (b->nsa) {
    b->off_lse3 = take(3 * B * H * N * 4);
    if (c.has_gate) b->off_dlogit = take(3 * B * H * N * 4);
    const CmpSplit sp = cmp_split(p);
    b->cmp_items = sp.items();
    if (p.n_cmp > 0) {
      b->off_dkc = take(B * Hkv * (size_t)p.ncmp_pad * d * 4);
      b->off_dvc = take(B * Hkv * (size_t)p.ncmp_pad * d * 4);
      b->off_clist = take(B * Hkv * (size_t)b->cmp_items * sp.chunk * 4);
      b->off_part = take(B * Hkv * (size_t)b->cmp_items * 2 * 128 * d * 4);
    }
  }
  if (b->lin) {
    b->off_dqacc = take(B * H * N * d * 4);    // linear-branch and gate part of dq (fp32)
    b->off_dkacc = take(B * Hkv * N * d * 4);  // linear-branch part of dk, dv (fp32)
    b->off_dvacc = take(B * Hkv * N * d * 4);
    b->off_drow = take(B * Hkv * (size_t)b->rows_t * p.dd * 2);         // [dS'_i | dZ_i] rows (bf16)
    b->off_maskt = take(B * Hkv * (size_t)p.nkb_pad * b->rows_t * 2);   // transposed aggregation mask
    b->off_dh = take(B * Hkv * (size_t)p.nkb * d * d * 2);              // dh'_j (bf16)
    b->off_dz = take(B * Hkv * (size_t)p.nkb * d * 4);                  // dz_j (fp32)
    if (c.has_proj)  // dW_p partial of each pair of key blocks (fp32)
      b->off_dwp = take(B * Hkv * (size_t)((p.nkb + 1) / 2) * d * d * 4);
    if (c.smooth_k) {  // column sums of the linear-branch dk: segment partials, then -sum / N_valid
      b->off_kcolp = take(B * Hkv * 64 * d * 4);
      b->off_kcol = take(B * Hkv * d * 4);
    }
  }
  b->total = off;
  return true;
}

enum BStage { kBZeroCols, kBDelta, kBLinear, kBMaskT, kBAggT, kBState, kBDq, kBDkdv, kBNsaPrep, kBDkdvCmp,
              kBCmpReduce };

static int bwd_stages_of(const Plan& p, const BwdPlan& bp, BStage* out) {
  int n = 0;
  out[n++] = kBZeroCols;
  if (bp.nsa) {
    // the compressed keys' gradients first: the token dK / dV kernel adds them
    out[n++] = kBNsaPrep;
    out[n++] = kBDq;
    if (p.n_cmp > 0) {
      out[n++] = kBDkdvCmp;
      out[n++] = kBCmpReduce;
    }
    out[n++] = kBDkdv;
    return n;
  }
  if (bp.lin) {
    out[n++] = kBLinear;
    out[n++] = kBMaskT;
    out[n++] = kBAggT;
    out[n++] = kBState;
  } else {
    out[n++] = kBDelta;
  }
  out[n++] = kBDq;
  out[n++] = kBDkdv;
  return n;
}

static const char* bwd_stage_name(BStage s) {
  switch (s) {
    case kBZeroCols: return "bwd_columns";
    case kBDelta: return "bwd_delta";
    case kBLinear: return "bwd_linear";
    case kBMaskT: return "bwd_mask_transpose";
    case kBAggT: return "bwd_aggregate_t";
    case kBState: return "bwd_state";
    case kBDq: return "bwd_flash_dq";
    case kBDkdv: return "bwd_flash_dkdv";
    case kBNsaPrep: return "bwd_nsa_prep";
    case kBDkdvCmp: return "bwd_flash_dkdv_cmp";
    case kBCmpReduce: return "bwd_cmp_reduce";
  }
  return "?";
}

static cudaError_t run_bwd_stage(BStage st, const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  switch (st) {
    case kBZeroCols: {
      // parameter gradients are sums of atomically added partials
      cudaError_t e = cudaSuccess;
      if (c.has_proj)
        e = cudaMemsetAsync(a.dw_p, 0, (size_t)(c.proj_per_head ? c.H : 1) * c.d * c.d * 4, s);
      if (e == cudaSuccess && c.has_gate)
        e = cudaMemsetAsync(a.dw_g, 0, (size_t)c.H * (c.nsa_branches ? 3 : 1) * c.d * 4, s);
      return e == cudaSuccess ? launch_cols(p, bp, a, s) : e;
    }
    case kBDelta: return launch_delta(p, bp, a, s);
    case kBLinear: return launch_lin_bwd(p, bp, a, s);
    case kBMaskT: return launch_mask_t(p, bp, a, s);
    case kBAggT: return launch_aggregate_t(p, bp, a, s);
    case kBState: return launch_state_bwd(p, bp, a, s);
    case kBDq: return launch_flash_dq(p, bp, a, s);
    case kBDkdv: return launch_flash_dkdv(p, bp, a, s);
    case kBNsaPrep: return launch_nsa_prep(p, bp, a, s);
    case kBDkdvCmp: return launch_flash_dkdv_cmp(p, bp, a, s);
    case kBCmpReduce: return launch_cmp_reduce(p, bp, a, s);
  }
  return cudaErrorInvalidValue;
}

static sla_status backward_impl(const void* q, const void* k, const void* v, const void* w_p, const void* w_g,
                                const sla_config* cfg, const void* out, const void* dout, void* dq, void* dk,
                                void* dv, float* dw_p, float* dw_g, const void* ws, size_t ws_bytes, void* bws,
                                size_t bws_bytes, void* stream, void* const* events, int32_t n_events) {
  const sla_status st = check_bwd_config(cfg);
  if (st != SLA_OK) return st;
  Plan p;
  BwdPlan bp;
  make_plan(cfg, &p);
  make_bwd_plan(p, &bp);
  const void* bf[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* x : bf)
    if (!x || !aligned(x, 16)) return SLA_ERR_INVALID_ARG;
  if (cfg->has_proj && (!w_p || !aligned(w_p, 16) || !dw_p || !aligned(dw_p, 16))) return SLA_ERR_INVALID_ARG;
  if (cfg->has_gate && (!w_g || !aligned(w_g, 16) || !dw_g || !aligned(dw_g, 16))) return SLA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return SLA_ERR_WORKSPACE;
  if (!bws || !aligned(bws, 256) || bws_bytes < bp.total) return SLA_ERR_WORKSPACE;
  BStage stages[9];
  const int ns = bwd_stages_of(p, bp, stages);
  if (events && n_events != ns + 1) return SLA_ERR_INVALID_ARG;
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.q = (const __nv_bfloat16*)q;
  a.k = (const __nv_bfloat16*)k;
  a.v = (const __nv_bfloat16*)v;
  a.w_p = (const __nv_bfloat16*)w_p;
  a.w_g = (const __nv_bfloat16*)w_g;
  a.out = (const __nv_bfloat16*)out;
  a.dout = (const __nv_bfloat16*)dout;
  a.dq = (__nv_bfloat16*)dq;
  a.dk = (__nv_bfloat16*)dk;
  a.dv = (__nv_bfloat16*)dv;
  a.dw_p = dw_p;
  a.dw_g = dw_g;
  a.ws = (const char*)ws;
  a.bws = (char*)bws;
  a.status = (int*)((char*)bws + bp.off_status);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(a.status, 0, 8, s) != cudaSuccess) return SLA_ERR_CUDA;
  if (events && cudaEventRecord((cudaEvent_t)events[0], s) != cudaSuccess) return SLA_ERR_CUDA;
  for (int i = 0; i < ns; ++i) {
    if (run_bwd_stage(stages[i], p, bp, a, s) != cudaSuccess) return SLA_ERR_CUDA;
    if (events && cudaEventRecord((cudaEvent_t)events[i + 1], s) != cudaSuccess) return SLA_ERR_CUDA;
  }
  return SLA_OK;
}

}  // namespace sla

using namespace sla;

extern "C" {

sla_status sla_validate_config(const sla_config* cfg) { return check_config(cfg); }

size_t sla_workspace_bytes(const sla_config* cfg) {
  Plan p;
  return make_plan(cfg, &p) ? p.total : 0;
}

sla_status sla_route(const void* q, const void* k, const sla_config* cfg, int8_t* mask_out,
                     int32_t* crit_idx, int32_t* neg_idx, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  sla_status st = check_config(cfg);
  if (st != SLA_OK) return st;
  make_plan(cfg, &p);
  if (!q || !k || !aligned(q, 16) || !aligned(k, 16)) return SLA_ERR_INVALID_ARG;
  const bool threeway = cfg->mode == SLA_MODE_THREEWAY;
  const int n_crit = threeway ? cfg->k_h : cfg->top_n;
  if (n_crit > 0 && (!crit_idx || !aligned(crit_idx, 4))) return SLA_ERR_INVALID_ARG;
  if (threeway && cfg->k_l > 0 && (!neg_idx || !aligned(neg_idx, 4))) return SLA_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return SLA_ERR_WORKSPACE;
  Args a;
  memset(&a, 0, sizeof(a));
  a.q = (const __nv_bfloat16*)q;
  a.k = (const __nv_bfloat16*)k;
  a.mask_out = mask_out;
  a.crit = n_crit > 0 ? crit_idx : nullptr;
  a.neg = threeway && cfg->k_l > 0 ? neg_idx : nullptr;
  a.ws = (char*)ws;
  a.status = (int*)((char*)ws + p.off_status);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(a.status, 0, 8, s) != cudaSuccess) return SLA_ERR_CUDA;
  return route_stages(p, a, s) == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

sla_status sla_forward(const void* q, const void* k, const void* v, const void* w_p,
                       const void* w_g, const sla_config* cfg, void* out, int8_t* mask_out,
                       void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(q, k, v, w_p, w_g, cfg, out, mask_out, ws, ws_bytes, stream, nullptr, 0);
}

sla_status sla_forward_blocks(const void* q, const void* k, const void* v, const void* w_p,
                              const void* w_g, const sla_config* cfg, int32_t qb_begin, int32_t qb_end,
                              void* out, int8_t* mask_out, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(q, k, v, w_p, w_g, cfg, out, mask_out, ws, ws_bytes, stream, nullptr, 0, qb_begin, qb_end);
}

sla_status sla_forward_timed(const void* q, const void* k, const void* v, const void* w_p,
                             const void* w_g, const sla_config* cfg, void* out, int8_t* mask_out,
                             void* ws, size_t ws_bytes, void* stream, void* const* events,
                             int32_t n_events) {
  if (!events) return SLA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, w_p, w_g, cfg, out, mask_out, ws, ws_bytes, stream, events,
                      n_events);
}

int32_t sla_num_stages(const sla_config* cfg) {
  Plan p;
  if (!make_plan(cfg, &p)) return -1;
  Stage st[kMaxStages];
  return stages_of(p, st);
}

const char* sla_stage_name(const sla_config* cfg, int32_t s) {
  Plan p;
  if (!make_plan(cfg, &p)) return nullptr;
  Stage st[kMaxStages];
  const int n = stages_of(p, st);
  return (s >= 0 && s < n) ? stage_name(st[s]) : nullptr;
}

sla_status sla_check_device_status(void* ws, void* stream, int32_t* detail) {
  if (!ws || !aligned(ws, 256)) return SLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SLA_ERR_CUDA;
  int st[2] = {0, 0};
  if (cudaMemcpy(st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return SLA_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(st)) != cudaSuccess) return SLA_ERR_CUDA;
  if (detail) *detail = st[1];
  if (st[0] == 0) return SLA_OK;
  if (st[0] == SLA_ERR_DEVICE_TIMEOUT || st[0] == SLA_ERR_DEVICE_CHECK) return (sla_status)st[0];
  return SLA_ERR_DEVICE_CHECK;
}

size_t sla_backward_workspace_bytes(const sla_config* cfg) {
  if (check_bwd_config(cfg) != SLA_OK) return 0;
  Plan p;
  BwdPlan bp;
  make_plan(cfg, &p);
  make_bwd_plan(p, &bp);
  return bp.total;
}

sla_status sla_backward(const void* q, const void* k, const void* v, const void* w_p, const void* w_g,
                        const sla_config* cfg, const void* out, const void* dout, void* dq, void* dk, void* dv,
                        float* dw_p, float* dw_g, const void* ws, size_t ws_bytes, void* bws, size_t bws_bytes,
                        void* stream) {
  return backward_impl(q, k, v, w_p, w_g, cfg, out, dout, dq, dk, dv, dw_p, dw_g, ws, ws_bytes, bws, bws_bytes,
                       stream, nullptr, 0);
}

sla_status sla_backward_timed(const void* q, const void* k, const void* v, const void* w_p, const void* w_g,
                              const sla_config* cfg, const void* out, const void* dout, void* dq, void* dk,
                              void* dv, float* dw_p, float* dw_g, const void* ws, size_t ws_bytes, void* bws,
                              size_t bws_bytes, void* stream, void* const* events, int32_t n_events) {
  if (!events) return SLA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, w_p, w_g, cfg, out, dout, dq, dk, dv, dw_p, dw_g, ws, ws_bytes, bws, bws_bytes,
                       stream, events, n_events);
}

int32_t sla_backward_num_stages(const sla_config* cfg) {
  if (check_bwd_config(cfg) != SLA_OK) return -1;
  Plan p;
  BwdPlan bp;
  make_plan(cfg, &p);
  make_bwd_plan(p, &bp);
  BStage st[9];
  return bwd_stages_of(p, bp, st);
}

const char* sla_backward_stage_name(const sla_config* cfg, int32_t s) {
  if (check_bwd_config(cfg) != SLA_OK) return nullptr;
  Plan p;
  BwdPlan bp;
  make_plan(cfg, &p);
  make_bwd_plan(p, &bp);
  BStage st[9];
  const int n = bwd_stages_of(p, bp, st);
  return (s >= 0 && s < n) ? bwd_stage_name(st[s]) : nullptr;
}

const char* sla_status_string(sla_status s) {
  switch (s) {
    case SLA_OK: return "ok";
    case SLA_ERR_INVALID_ARG: return "invalid argument";
    case SLA_ERR_UNSUPPORTED: return "configuration not supported by the kernels";
    case SLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SLA_ERR_CUDA: return "CUDA runtime or launch error";
    case SLA_ERR_DEVICE_TIMEOUT: return "device-side bounded wait ran out";
    case SLA_ERR_DEVICE_CHECK: return "device-side range check failed";
  }
  return "unknown status";
}

const char* sla_version(void) { return "0.1.0"; }

}  // extern "C"
