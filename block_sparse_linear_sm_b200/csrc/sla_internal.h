// Internal host-side interface between the C ABI (sla_api.cu) and the kernels.
#pragma once
#include <cuda.h>  // CUtensorMap (type only)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sla.h"

namespace sla {

constexpr int kBlock = 64;
constexpr int kMaxBlocks = 4096;  // nkb limit of the routing sort (N <= 262144)

// Device status word: status[0] = sla_status code, status[1] = detail.
enum DeviceDetail : int {
  kDetailFlashIndex = 101,      // flash kernel read a block index outside [0, nkb)
  kDetailRouteSelect = 102,    // the exact class-boundary selection lost a block (broken invariant)
  kDetailFlashAlign = 103,     // shared-memory base not 1024-byte aligned
  kDetailTimeout = 200,
  kDetailSelftest = 300,       // the failure-detection self-test's wait ran out (expected)
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Derived sizes and the workspace carve-up for one configuration.
struct Plan {
  sla_config c;
  int nqb, nkb, group;
  int nqb_pad, nkb_pad;  // aggregation GEMM padding (128 rows, 64 columns)
  int dd;                // row length of the per-block linear state: d*d + d, padded to 128
  float scale;
  // byte offsets into ws
  size_t off_status, off_qbar, off_kbar, off_scores, off_kflag, off_crit, off_neg, off_mmask, off_hs, off_ss,
      off_zs, off_phiq, off_gate, off_kmean, off_lse, total;
  // NSA's branches (top-n mode): compressed K, V [B*H_kv][ncmp_pad][d] and the three
  // branch outputs [B*H][N][d] (bf16); off_lse then holds three rows [3][B*H][N]
  // (compressed, selected, window)
  int n_cmp, ncmp_pad;
  size_t off_kc, off_vc, off_oc, off_os, off_ow;
  // query blocks whose output rows this call writes: [qb0, qb1) (the whole layer by
  // default; sla_forward_blocks narrows it, qb0 even)
  int qb0, qb1;
};

bool make_plan(const sla_config* c, Plan* p);

// process-unique id of the current CUDA context, 0 if it cannot be read (noalloc.cu)
unsigned long long current_context_id();
// sla_forward without the internal side stream (callers that run several layers on their
// own streams at once, where one shared side stream would serialise them)
sla_status forward_single_stream(const void* q, const void* k, const void* v, const void* w_p, const void* w_g,
                                 const sla_config* cfg, void* out, int8_t* mask_out, void* ws, size_t ws_bytes,
                                 void* stream);

// Raw pointers of one launch.
struct Args {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* w_p;
  const __nv_bfloat16* w_g;
  __nv_bfloat16* out;
  int8_t* mask_out;
  int32_t* crit;      // THREEWAY critical lists / TOPN selected lists
  int32_t* neg;       // THREEWAY negligible lists (may be null)
  char* ws;
  int* status;
};

// 3D bf16 TMA tensor map [d2][d1][d0] (d0 innermost) with byte strides s1, s2,
// box (b0, b1, 1) and 128-byte swizzle; out-of-range elements read as zero.
// Defined in tmap.cu; false if the driver entry point or the encode fails.
bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1);

// kernel launchers (return the launch error)
cudaError_t launch_pool(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_kcos(const Plan& p, const Args& a, cudaStream_t s);  // cos_filter flags
// the routing stages alone (sla_route, sla_route_noalloc): lists and mask, no aggregation mask
cudaError_t route_stages(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_scores(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_classify(const Plan& p, const Args& a, bool write_mmask, cudaStream_t s);
cudaError_t launch_select(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_state(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_aggregate(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_flash(const Plan& p, const Args& a, cudaStream_t s);
cudaError_t launch_flash_nsa(const Plan& p, const Args& a, int branch, cudaStream_t s);  // 1 cmp, 2 slc, 3 win
cudaError_t launch_compress(const Plan& p, const Args& a, cudaStream_t s);

// ---------------------------------------------------------------------------
// backward pass (three-way mode)
// ---------------------------------------------------------------------------
// Carve-up of the backward scratch (bws). nqb_pad rows per query head of a KV
// group form the K extent of the transposed aggregation.
struct BwdPlan {
  bool lin;       // the layer has a linear branch
  bool nsa;       // NSA's three branches
  int rows_t;     // group * nqb_pad
  int words;      // 32-bit words of one column bitmap (query blocks)
  int cmp_items;  // NSA: work items of the compressed-key dK / dV kernel per KV head
  size_t off_status, off_delta, off_dqacc, off_dkacc, off_dvacc, off_drow, off_maskt, off_dh, off_dz,
      off_dwp, off_kcolp, off_kcol, off_bits, off_dlist, total;
  size_t off_ctr;  // unit counters of the persistent flash kernels (dQ, dK / dV, compressed-key dK / dV)
  size_t off_lbits;  // top-n modes: the dK / dV loader's four query-block bitmaps per unit
  // NSA: per-branch log-sum-exp with the gate folded in [3][B*H][N], gate-logit gradients
  // [3][B*H][N], compressed-key gradients dKc, dVc [B*H_kv][ncmp_pad][d] (fp32), the
  // compressed-key kernel's lists and raw partials
  size_t off_lse3, off_dlogit, off_dkc, off_dvc, off_clist, off_part;
};
bool make_bwd_plan(const Plan& p, BwdPlan* b);

// NSA's compressed keys: the (query head, query block) entries of the pair of compressed
// tiles u (keys 128 u .. 128 u + 127) are every query head of the group times the query
// blocks i >= first(u), the first block with a row t = 64 i + 63 that attends key 128 u
// (128 u * stride + span <= t); they are cut into chunks of `chunk` entries. Host and
// device share this arithmetic.
struct CmpSplit {
  int n_cmp, kstride, kspan, nqb, group, chunk;
  __host__ __device__ int first_block(int u) const {
    const long long need = (long long)128 * u * kstride + kspan - (kBlock - 1);
    return need <= 0 ? 0 : (int)((need + kBlock - 1) / kBlock);
  }
  __host__ __device__ int entries(int u) const {
    if (128 * u >= n_cmp) return 0;
    const int f = first_block(u);
    return f >= nqb ? 0 : group * (nqb - f);
  }
  __host__ __device__ int chunks(int u) const { return (entries(u) + chunk - 1) / chunk; }
  __host__ __device__ int units() const { return (n_cmp + 127) / 128; }
  __host__ __device__ int items() const {
    int n = 0;
    for (int u = 0; u < units(); ++u) n += chunks(u);
    return n;
  }
};

CmpSplit cmp_split(const Plan& p);
int dkdv_list_cap(const Plan& p);

struct BwdArgs {
  const __nv_bfloat16 *q, *k, *v, *w_p, *w_g, *out, *dout;
  __nv_bfloat16 *dq, *dk, *dv;
  float *dw_p, *dw_g;
  const char* ws;  // the forward pass's workspace (read only)
  char* bws;       // backward scratch
  int* status;     // in bws
};

cudaError_t launch_delta(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_lin_bwd(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_mask_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_aggregate_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_state_bwd(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_cols(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_flash_dq(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_flash_dkdv(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
// NSA's branches
cudaError_t launch_nsa_prep(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_flash_dkdv_cmp(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_cmp_reduce(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);

}  // namespace sla
