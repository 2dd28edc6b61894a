// Router kernels: block pooling, pooled scores and per-row routing.
//
// Block pooling and pooled scores follow the SLA analysis page (arXiv
// 2509.24006, compressed attention prediction: mean pooling to an (N/b)^2
// block problem) and the 2025 sparse-attention review, section 11
// (SpargeAttn prediction: q_i = mean(Q_i), k_j = mean(K_j), S_hat = q k^T,
// P_hat = softmax). The three-way split is the SLA critical / marginal /
// negligible classification by TopK / BottomK; the top-n mode is the MoBA /
// NSA block selection (2025 review, section 4; sparse attention survey,
// section 2, NSA selected branch).
//
// Pooling and scores are computed in float64 so that the block order, which
// decides integers (the classes), is exact up to summation order.
#include "common.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// pooling: one CTA per (head row, block); d/2 threads, two columns each.
// Q heads first (B*H of them), then KV heads (B*H_kv).
// ---------------------------------------------------------------------------
__global__ void pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                            double* __restrict__ qbar, double* __restrict__ kbar, int n_qheads,
                            int N, int n_valid, int d, int nb) {
  const int j = blockIdx.x;
  const int hrow = blockIdx.y;
  const bool is_q = hrow < n_qheads;
  const int hh = is_q ? hrow : hrow - n_qheads;
  const __nv_bfloat16* x = (is_q ? q : k) + ((size_t)hh * N + (size_t)j * kBlock) * d;
  double* out = (is_q ? qbar : kbar) + ((size_t)hh * nb + j) * d;
  const int c = threadIdx.x * 2;
  int nv = n_valid - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  double s0 = 0.0, s1 = 0.0;
#pragma unroll 8
  for (int t = 0; t < nv; ++t) {
    uint32_t u = *reinterpret_cast<const uint32_t*>(x + (size_t)t * d + c);
    float2 f = unpack_bf16(u);
    s0 += (double)f.x;
    s1 += (double)f.y;
  }
  // mean = sum / count (one rounding, as a division)
  out[c] = nv > 0 ? s0 / (double)nv : 0.0;
  out[c + 1] = nv > 0 ? s1 / (double)nv : 0.0;
}

cudaError_t launch_pool(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  double* qbar = reinterpret_cast<double*>(a.ws + p.off_qbar);
  double* kbar = reinterpret_cast<double*>(a.ws + p.off_kbar);
  dim3 grid(p.nqb, c.B * c.H + c.B * c.H_kv);
  pool_kernel<<<grid, c.d / 2, 0, s>>>(a.q, a.k, qbar, kbar, c.B * c.H, c.N, c.N_valid, c.d, p.nqb);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pooled scores: s[bh][i][j] = scale * qbar[bh][i] . kbar[bkv][j], float64.
// 64x64 output tile per CTA, 256 threads with 4x4 outputs each, K chunks of 16.
// In top-n mode only j < i is ever read, so tiles wholly above the diagonal
// are skipped.
// ---------------------------------------------------------------------------
constexpr int kSTile = 64;
constexpr int kSK = 16;

__global__ void __launch_bounds__(256) scores_kernel(const double* __restrict__ qbar,
                                                     const double* __restrict__ kbar,
                                                     double* __restrict__ scores, int H, int group,
                                                     int nb, int d, double scale, int lower_only) {
  const int bh = blockIdx.z;
  const int b = bh / H, h = bh % H;
  const int bkv = b * (H / group) + h / group;
  const int i0 = blockIdx.y * kSTile, j0 = blockIdx.x * kSTile;
  if (lower_only && j0 > i0 + kSTile - 1) return;
  __shared__ double As[kSK][kSTile + 1];
  __shared__ double Bs[kSK][kSTile + 1];
  const double* A = qbar + (size_t)bh * nb * d;
  const double* Bm = kbar + (size_t)bkv * nb * d;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kSK) {
    for (int e = threadIdx.x; e < kSTile * kSK; e += 256) {
      const int r = e / kSK, kk = e % kSK;
      const int ia = i0 + r, jb = j0 + r;
      As[kk][r] = ia < nb ? A[(size_t)ia * d + k0 + kk] : 0.0;
      Bs[kk][r] = jb < nb ? Bm[(size_t)jb * d + k0 + kk] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      double av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        av[u] = As[kk][ty + 16 * u];
        bv[u] = Bs[kk][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fma(av[u], bv[w], acc[u][w]);
    }
    __syncthreads();
  }
  double* S = scores + (size_t)bh * nb * nb;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty + 16 * u;
    if (i >= nb) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = j0 + tx + 16 * w;
      if (j < nb) S[(size_t)i * nb + j] = acc[u][w] * scale;
    }
  }
}

cudaError_t launch_scores(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* qbar = reinterpret_cast<const double*>(a.ws + p.off_qbar);
  const double* kbar = reinterpret_cast<const double*>(a.ws + p.off_kbar);
  double* sc = reinterpret_cast<double*>(a.ws + p.off_scores);
  const int t = (p.nqb + kSTile - 1) / kSTile;
  dim3 grid(t, t, c.B * c.H);
  scores_kernel<<<grid, 256, 0, s>>>(qbar, kbar, sc, c.H, p.group, p.nqb, c.d, (double)p.scale,
                                     c.mode == SLA_MODE_TOPN_WINDOW);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// sorting helpers: order-preserving 64-bit key of a double, bitonic sort of
// (key, index) pairs so that higher keys come first and equal keys keep the
// lower index first.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long order_key(double x) {
  const long long b = __double_as_longlong(x);
  return b < 0 ? ~(unsigned long long)b : ((unsigned long long)b | 0x8000000000000000ull);
}

__device__ __forceinline__ bool ranks_before(unsigned long long ka, int ia, unsigned long long kb,
                                             int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// Sorts P (a power of two) pairs in shared memory; all threads of the CTA take part.
__device__ void bitonic_sort(unsigned long long* key, uint16_t* idx, int P) {
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int l = i ^ j;
        if (l > i) {
          const bool first_half = (i & k) == 0;
          const bool i_first = ranks_before(key[i], idx[i], key[l], idx[l]);
          if (first_half != i_first) {
            unsigned long long tk = key[i];
            key[i] = key[l];
            key[l] = tk;
            uint16_t ti = idx[i];
            idx[i] = idx[l];
            idx[l] = ti;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Block-wide exclusive scan of one int per thread; returns the prefix, *total gets the sum.
__device__ int block_exclusive_scan(int v, int* total, int* scratch /* >= 33 ints */) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) scratch[lane] = w;
    if (lane == nw - 1) scratch[32] = w;
  }
  __syncthreads();
  const int before = (wid > 0 ? scratch[wid - 1] : 0) + x - v;
  *total = scratch[32];
  __syncthreads();
  return before;
}

// Writes the ascending list of indices j < n with cls[j] == want into out.
__device__ void compact_ascending(const int8_t* cls, int n, int8_t want, int32_t* out,
                                  int* scratch) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per;
  const int hi = min(lo + per, n);
  int cnt = 0;
  for (int j = lo; j < hi; ++j) cnt += cls[j] == want;
  int total;
  int pos = block_exclusive_scan(cnt, &total, scratch);
  for (int j = lo; j < hi; ++j)
    if (cls[j] == want) out[pos++] = j;
}

// ---------------------------------------------------------------------------
// three-way classification: one CTA per (b, h, query block i).
// ---------------------------------------------------------------------------
constexpr int kSortThreads = 256;

__global__ void __launch_bounds__(kSortThreads) classify_kernel(
    const double* __restrict__ scores, int8_t* __restrict__ mask_out, int32_t* __restrict__ crit,
    int32_t* __restrict__ neg, __nv_bfloat16* __restrict__ mmask, int nb, int P, int k_h, int k_l,
    int nkb_pad, int nqb_pad) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);
  uint16_t* idx = reinterpret_cast<uint16_t*>(smem + (size_t)P * 8);
  int8_t* cls = reinterpret_cast<int8_t*>(smem + (size_t)P * 10);
  __shared__ int scratch[33];
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  if (i >= nb) {
    // rows past the last query block of the aggregation mask are zero
    __nv_bfloat16* mrow = mmask + ((size_t)bh * nqb_pad + i) * nkb_pad;
    for (int j = threadIdx.x; j < nkb_pad; j += blockDim.x) mrow[j] = __float2bfloat16(0.f);
    return;
  }
  const double* row = scores + ((size_t)bh * nb + i) * nb;
  for (int j = threadIdx.x; j < P; j += blockDim.x) {
    key[j] = j < nb ? order_key(row[j]) : 0ull;
    idx[j] = (uint16_t)(j < nb ? j : 0xFFFF);
  }
  __syncthreads();
  bitonic_sort(key, idx, P);
  for (int p = threadIdx.x; p < nb; p += blockDim.x)
    cls[idx[p]] = p < k_h ? (int8_t)2 : (p >= nb - k_l ? (int8_t)0 : (int8_t)1);
  __syncthreads();
  const size_t rowoff = ((size_t)bh * nb + i) * nb;
  if (mask_out)
    for (int j = threadIdx.x; j < nb; j += blockDim.x) mask_out[rowoff + j] = cls[j];
  if (mmask) {
    __nv_bfloat16* mrow = mmask + ((size_t)bh * nqb_pad + i) * nkb_pad;
    for (int j = threadIdx.x; j < nkb_pad; j += blockDim.x)
      mrow[j] = __float2bfloat16(j < nb && cls[j] == 1 ? 1.f : 0.f);
  }
  if (crit && k_h > 0) compact_ascending(cls, nb, 2, crit + ((size_t)bh * nb + i) * k_h, scratch);
  if (neg && k_l > 0) compact_ascending(cls, nb, 0, neg + ((size_t)bh * nb + i) * k_l, scratch);
}

static int pow2_at_least(int n) {
  int P = 1;
  while (P < n) P <<= 1;
  return P;
}

cudaError_t launch_classify(const Plan& p, const Args& a, bool write_mmask, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* sc = reinterpret_cast<const double*>(a.ws + p.off_scores);
  __nv_bfloat16* mm = write_mmask ? reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_mmask) : nullptr;
  const int P = pow2_at_least(p.nkb);
  const size_t smem = (size_t)P * 10 + align_up(p.nkb, 16);
  cudaError_t e = cudaFuncSetAttribute(classify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // with the aggregation mask, extra CTAs zero its padding rows nqb..nqb_pad
  dim3 grid(write_mmask ? p.nqb_pad : p.nqb, c.B * c.H);
  classify_kernel<<<grid, kSortThreads, smem, s>>>(sc, a.mask_out, a.crit, a.neg, mm, p.nkb, P,
                                                   c.k_h, c.k_l, p.nkb_pad, p.nqb_pad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// top-n selection: one CTA per (b, KV head, query block i). The group's heads
// each take a softmax of their pooled scores over the past blocks j < i; the
// probabilities are summed and the top min(top_n, i) kept.
// ---------------------------------------------------------------------------
__device__ double block_reduce(double v, bool is_max, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    double y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmax(v, y) : v + y;
  }
  if (lane == 0) red[wid] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = is_max ? fmax(r, red[w]) : r + red[w];
    red[32] = r;
  }
  __syncthreads();
  double r = red[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSortThreads) select_kernel(const double* __restrict__ scores,
                                                              int8_t* __restrict__ mask_out,
                                                              int32_t* __restrict__ sel, int H,
                                                              int group, int nb, int top_n,
                                                              int pmax) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int i = blockIdx.x;
  const int bkv = blockIdx.y;
  const int Hkv = H / group;
  const int b = bkv / Hkv, hk = bkv % Hkv;
  int P = 1;
  while (P < i) P <<= 1;
  double* prob = reinterpret_cast<double*>(smem);
  // prob: nb doubles; key: pmax (a power of two >= nb) keys; idx: pmax indices
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem + (size_t)nb * 8);
  uint16_t* idx = reinterpret_cast<uint16_t*>(smem + (size_t)nb * 8 + (size_t)pmax * 8);
  __shared__ double red[33];
  __shared__ int chosen[64 + 1];
  for (int j = threadIdx.x; j < i; j += blockDim.x) prob[j] = 0.0;
  __syncthreads();
  for (int g = 0; g < group && i > 0; ++g) {
    const int h = hk * group + g;
    const double* row = scores + (((size_t)b * H + h) * nb + i) * nb;
    double m = -INFINITY;
    for (int j = threadIdx.x; j < i; j += blockDim.x) m = fmax(m, row[j]);
    m = block_reduce(m, true, red);
    double sum = 0.0;
    for (int j = threadIdx.x; j < i; j += blockDim.x) sum += exp(row[j] - m);
    sum = block_reduce(sum, false, red);
    const double inv = 1.0 / sum;
    for (int j = threadIdx.x; j < i; j += blockDim.x) prob[j] += exp(row[j] - m) * inv;
    __syncthreads();
  }
  const int n = i < top_n ? i : top_n;
  if (i > 0) {
    for (int j = threadIdx.x; j < P; j += blockDim.x) {
      key[j] = j < i ? order_key(prob[j]) : 0ull;
      idx[j] = (uint16_t)(j < i ? j : 0xFFFF);
    }
    __syncthreads();
    bitonic_sort(key, idx, P);
  }
  // ascending order of the chosen blocks: count how many chosen indices are smaller
  if (threadIdx.x < n) {
    const int me = idx[threadIdx.x];
    int r = 0;
    for (int u = 0; u < n; ++u) r += idx[u] < me;
    chosen[r] = me;
  }
  __syncthreads();
  const size_t rowid = (size_t)bkv * nb + i;
  for (int u = threadIdx.x; u < top_n; u += blockDim.x) sel[rowid * top_n + u] = u < n ? chosen[u] : -1;
  if (mask_out) {
    for (int j = threadIdx.x; j < nb; j += blockDim.x) mask_out[rowid * nb + j] = 0;
    __syncthreads();
    if (threadIdx.x < n) mask_out[rowid * nb + chosen[threadIdx.x]] = 2;
  }
}

cudaError_t launch_select(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* sc = reinterpret_cast<const double*>(a.ws + p.off_scores);
  // the sort arrays hold a power of two >= i < nkb elements
  const int P = pow2_at_least(p.nkb);
  const size_t use = (size_t)p.nkb * 8 + (size_t)P * 10 + 16;
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)use);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nqb, c.B * c.H_kv);
  select_kernel<<<grid, kSortThreads, use, s>>>(sc, a.mask_out, a.crit, c.H, p.group, p.nkb,
                                                c.top_n, P);
  return cudaGetLastError();
}

}  // namespace sla
