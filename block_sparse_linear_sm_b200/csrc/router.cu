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
// Q heads first (B*H of them), then KV heads (B*H_kv). For layers with a linear
// branch the Q pass also writes phi(Q) (bf16, the left factor of the linear
// branch's numerator and denominator) and, with a gate, g_t = sigmoid(q_t .
// w_g[h]) per token: Q is read here anyway, so the epilogue need not
// transform it again.
// ---------------------------------------------------------------------------
__global__ void pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                            double* __restrict__ qbar, double* __restrict__ kbar, int n_qheads,
                            int N, int n_valid, int d, int nb, __nv_bfloat16* __restrict__ phiq,
                            const __nv_bfloat16* __restrict__ w_g, float* __restrict__ gate, int H) {
  const int j = blockIdx.x;
  const int hrow = blockIdx.y;
  const bool is_q = hrow < n_qheads;
  const int hh = is_q ? hrow : hrow - n_qheads;
  const __nv_bfloat16* x = (is_q ? q : k) + ((size_t)hh * N + (size_t)j * kBlock) * d;
  double* out = (is_q ? qbar : kbar) + ((size_t)hh * nb + j) * d;
  const int c = threadIdx.x * 2;
  int nv = n_valid - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  __nv_bfloat16* fq =
      (is_q && phiq) ? phiq + ((size_t)hh * N + (size_t)j * kBlock) * d : nullptr;
  double s0 = 0.0, s1 = 0.0;
#pragma unroll 8
  for (int t = 0; t < nv; ++t) {
    uint32_t u = *reinterpret_cast<const uint32_t*>(x + (size_t)t * d + c);
    float2 f = unpack_bf16(u);
    s0 += (double)f.x;
    s1 += (double)f.y;
    if (fq) *reinterpret_cast<uint32_t*>(fq + (size_t)t * d + c) = pack_bf16(phi(f.x), phi(f.y));
  }
  // mean = sum / count (one rounding, as a division)
  out[c] = nv > 0 ? s0 / (double)nv : 0.0;
  out[c + 1] = nv > 0 ? s1 / (double)nv : 0.0;
  if (is_q && gate) {
    // one token per thread; the rows were just read, so they come from cache
    const __nv_bfloat16* wg = w_g + (size_t)(hh % H) * d;
    for (int t = threadIdx.x; t < nv; t += blockDim.x) {
      const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)t * d);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c8 = 0; c8 < d / 8; ++c8) {
        const uint4 u = row[c8];
        const uint4 w = *reinterpret_cast<const uint4*>(wg + c8 * 8);
        const uint32_t* uu = reinterpret_cast<const uint32_t*>(&u);
        const uint32_t* ww = reinterpret_cast<const uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fu = unpack_bf16(uu[e]), fw = unpack_bf16(ww[e]);
          acc[e] = fmaf(fu.x, fw.x, fmaf(fu.y, fw.y, acc[e]));
        }
      }
      const float dot = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      gate[(size_t)hh * N + (size_t)j * kBlock + t] = 1.f / (1.f + __expf(-dot));
    }
  }
}

// ---------------------------------------------------------------------------
// key-block similarity (2025 review, section 11, SpargeAttn: s_kj = CosSim(K_j),
// S_hat[i, j] = -inf when s_kj < theta): one warp per (KV head row, block);
// CosSim = |sum_t k_t / |k_t||^2 / n^2 over the n valid tokens, in float64 like
// the pooled means (a zero token counts as the zero vector). Each token is
// handled by D/32 lanes holding 32 columns each, 32/(D/32) tokens at a time;
// each lane keeps the running sum of its 32 columns of the normalised tokens.
// Writes 1 for the blocks below theta.
// ---------------------------------------------------------------------------
template <int D>
__global__ void kcos_kernel(const __nv_bfloat16* __restrict__ k, uint8_t* __restrict__ kflag, int rows,
                            int nb, int N, int n_valid, double theta) {
  constexpr int LPT = D / 32;        // lanes per token
  constexpr int TPI = 32 / LPT;      // tokens per iteration
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= rows) return;
  const int bkv = wid / nb, j = wid % nb;
  const int sub = lane % LPT, tk = lane / LPT;  // column part, token slot
  int nv = n_valid - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  const uint4* x = reinterpret_cast<const uint4*>(k + ((size_t)bkv * N + (size_t)j * kBlock) * D) + sub * 4;
  double acc[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) acc[e] = 0.0;
  for (int t0 = 0; t0 < nv; t0 += TPI) {
    const int t = t0 + tk;
    float f[32];
    if (t < nv) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 u = x[(size_t)t * (D / 8) + c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = unpack_bf16(w[e]);
          f[8 * c + 2 * e] = v.x;
          f[8 * c + 2 * e + 1] = v.y;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) f[e] = 0.f;
    }
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fma((double)f[e], (double)f[e], ss);
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // the token's lanes
    if (ss > 0.0) {
      const double inv = 1.0 / sqrt(ss);
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[e] = fma((double)f[e], inv, acc[e]);
    }
  }
  // add the token slots' sums (lanes with the same column part), then |sum|^2
  double sq = 0.0;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    double v = acc[e];
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    sq = fma(v, v, sq);
  }
  // lanes 0 .. LPT-1 now hold the column parts' shares
#pragma unroll
  for (int o = 1; o < LPT; o <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0) kflag[wid] = nv > 0 && sq / ((double)nv * (double)nv) < theta ? 1 : 0;
}

cudaError_t launch_pool(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  double* qbar = reinterpret_cast<double*>(a.ws + p.off_qbar);
  double* kbar = reinterpret_cast<double*>(a.ws + p.off_kbar);
  // phi(Q) and the gate feed the linear branch of a forward pass; routing-only
  // calls (no V) do not produce them
  const bool lin =
      a.v != nullptr && c.mode == SLA_MODE_THREEWAY && (p.nkb - c.k_h - c.k_l > 0 || c.linear_all);
  __nv_bfloat16* phiq = lin ? reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_phiq) : nullptr;
  float* gate = (lin && c.has_gate) ? reinterpret_cast<float*>(a.ws + p.off_gate) : nullptr;
  dim3 grid(p.nqb, c.B * c.H + c.B * c.H_kv);
  pool_kernel<<<grid, c.d / 2, 0, s>>>(a.q, a.k, qbar, kbar, c.B * c.H, c.N, c.N_valid, c.d,
                                       p.nqb, phiq, gate ? a.w_g : nullptr, gate, c.H);
  cudaError_t e = cudaGetLastError();
  // part of routing: the filter flags feed classify / select
  if (e != cudaSuccess || !c.cos_filter) return e;
  return launch_kcos(p, a, s);
}

cudaError_t launch_kcos(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const int rows = c.B * c.H_kv * p.nkb;
  uint8_t* kflag = reinterpret_cast<uint8_t*>(a.ws + p.off_kflag);
  const int blocks = (rows + 3) / 4;  // four warps (blocks) per CTA
  if (c.d == 128)
    kcos_kernel<128><<<blocks, 128, 0, s>>>(a.k, kflag, rows, p.nkb, c.N, c.N_valid, (double)c.cos_theta);
  else
    kcos_kernel<64><<<blocks, 128, 0, s>>>(a.k, kflag, rows, p.nkb, c.N, c.N_valid, (double)c.cos_theta);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pooled scores: s[bh][i][j] = scale * qbar[bh][i] . kbar[bkv][j], float64,
// on the FP64 tensor-core path (mma.sync m8n8k4, fp64 in and out; every product
// and sum is an IEEE double operation). 64 x 64 output tile per CTA, four warps
// of 32 x 32 (4 x 4 fragments of 8 x 8), K chunks of 16. In top-n mode only
// j < i is ever read, so tiles wholly above the diagonal are skipped.
// ---------------------------------------------------------------------------
constexpr int kSTile = 64;
constexpr int kSK = 16;       // k columns per pipeline stage
constexpr int kSPad = 20;     // doubles per shared-memory row: a fragment read takes two wavefronts
constexpr int kSStages = 4;   // cp.async ring depth
constexpr int kScoresSmem = kSStages * 2 * kSTile * kSPad * 8;

__device__ __forceinline__ void dmma_8x8x4(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(128) scores_kernel(const double* __restrict__ qbar,
                                                     const double* __restrict__ kbar,
                                                     double* __restrict__ scores, int H, int group,
                                                     int nb, int d, double scale, int lower_only) {
  const int bh = blockIdx.z;
  const int b = bh / H, h = bh % H;
  const int bkv = b * (H / group) + h / group;
  const int i0 = blockIdx.y * kSTile, j0 = blockIdx.x * kSTile;
  if (lower_only && j0 > i0 + kSTile - 1) return;
  // stage s: A rows [kSTile][kSPad], then B rows; k chunks arrive by cp.async
  extern __shared__ __align__(16) double ssm[];
  const double* A = qbar + (size_t)bh * nb * d;
  const double* Bm = kbar + (size_t)bkv * nb * d;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int wi = (w >> 1) * 32, wj = (w & 1) * 32;  // warp tile origin
  const int nk = d / kSK;
  auto load = [&](int kc, int st) {
    double* As = ssm + (size_t)st * 2 * kSTile * kSPad;
    double* Bs = As + kSTile * kSPad;
    // 64 rows x 8 sixteen-byte pieces per matrix; rows past nb are zero-filled
    for (int e = tid; e < kSTile * 8; e += 128) {
      const int r = e >> 3, pc = e & 7;
      const int ia = i0 + r, jb = j0 + r;
      cp_async16(smem_u32(As + r * kSPad + 2 * pc), A + (size_t)(ia < nb ? ia : 0) * d + kc * kSK + 2 * pc,
                 ia < nb ? 16 : 0);
      cp_async16(smem_u32(Bs + r * kSPad + 2 * pc), Bm + (size_t)(jb < nb ? jb : 0) * d + kc * kSK + 2 * pc,
                 jb < nb ? 16 : 0);
    }
  };
#pragma unroll
  for (int st = 0; st < kSStages - 1; ++st) {
    if (st < nk) load(st, st);
    cp_async_commit();
  }
  double acc[4][4][2] = {};
  for (int kc = 0; kc < nk; ++kc) {
    cp_async_wait<kSStages - 2>();
    __syncthreads();  // chunk kc landed for everyone; stage (kc - 1) % S is free again
    if (kc + kSStages - 1 < nk) load(kc + kSStages - 1, (kc + kSStages - 1) % kSStages);
    cp_async_commit();
    const double* As = ssm + (size_t)(kc % kSStages) * 2 * kSTile * kSPad;
    const double* Bs = As + kSTile * kSPad;
#pragma unroll
    for (int k4 = 0; k4 < kSK; k4 += 4) {
      double af[4], bf[4];
      // A fragment: row lane/4, column lane%4; B fragment: row (k) lane%4, column lane/4
#pragma unroll
      for (int m = 0; m < 4; ++m) af[m] = As[(wi + 8 * m + (lane >> 2)) * kSPad + k4 + (lane & 3)];
#pragma unroll
      for (int n = 0; n < 4; ++n) bf[n] = Bs[(wj + 8 * n + (lane >> 2)) * kSPad + k4 + (lane & 3)];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n) dmma_8x8x4(acc[m][n], af[m], bf[n]);
    }
  }
  double* S = scores + (size_t)bh * nb * nb;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int i = i0 + wi + 8 * m + (lane >> 2);
    if (i >= nb) continue;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int j = j0 + wj + 8 * n + 2 * (lane & 3);
      if (j < nb) S[(size_t)i * nb + j] = acc[m][n][0] * scale;
      if (j + 1 < nb) S[(size_t)i * nb + j + 1] = acc[m][n][1] * scale;
    }
  }
}

cudaError_t launch_scores(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* qbar = reinterpret_cast<const double*>(a.ws + p.off_qbar);
  const double* kbar = reinterpret_cast<const double*>(a.ws + p.off_kbar);
  double* sc = reinterpret_cast<double*>(a.ws + p.off_scores);
  const int t = (p.nqb + kSTile - 1) / kSTile;
  cudaError_t e = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoresSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(t, t, c.B * c.H);
  scores_kernel<<<grid, 128, kScoresSmem, s>>>(qbar, kbar, sc, c.H, p.group, p.nqb, c.d, (double)p.scale,
                                               c.mode == SLA_MODE_TOPN_WINDOW);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Exact top-c selection, one warp per row.
//
// Scores become order-preserving 64-bit keys; "j ranks before l" means
// key_j > key_l, or equal keys and j < l (the lower block index first). The
// top c of a row are found by an MSD radix select over 8-bit digits: each pass
// histograms the digit of the keys that still share the selected prefix and
// picks the bin holding the c-th key. The pass stops early once that bin is
// taken whole; after all 8 digits, keys equal to the boundary key are taken in
// index order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long order_key(double x) {
  const long long b = __double_as_longlong(x);
  return b < 0 ? ~(unsigned long long)b : ((unsigned long long)b | 0x8000000000000000ull);
}

struct TopSel {
  unsigned long long prefix, mask;  // keys with (key & mask) > prefix are in the set
  int need;                         // how many keys with (key & mask) == prefix are in
  bool whole;                       // all keys with (key & mask) == prefix are in
};

// keys[0..n) in shared memory, hist = 256 words of this warp; 1 <= c <= n.
__device__ TopSel warp_select_top(const unsigned long long* keys, int n, int c, unsigned* hist) {
  const int lane = threadIdx.x & 31;
  TopSel r{0ull, 0ull, c, false};
  for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) hist[lane * 8 + u] = 0u;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const unsigned long long key = keys[j];
      if ((key & r.mask) == r.prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending)
    unsigned cnt[8];
    unsigned tot = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cnt[u] = hist[255 - 8 * lane - u];
      tot += cnt[u];
    }
    unsigned incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned excl = incl - tot;
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)r.need);
    const int owner = __ffs(hit) - 1;
    int bin = 0;
    unsigned above = 0, inbin = 0;
    if (lane == owner) {
      unsigned run = excl;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (run + cnt[u] >= (unsigned)r.need) {
          bin = 255 - 8 * lane - u;
          above = run;
          inbin = cnt[u];
          break;
        }
        run += cnt[u];
      }
    }
    bin = __shfl_sync(0xffffffffu, bin, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    inbin = __shfl_sync(0xffffffffu, inbin, owner);
    __syncwarp();
    r.need -= (int)above;
    r.prefix |= (unsigned long long)bin << shift;
    r.mask |= 255ull << shift;
    if (inbin == (unsigned)r.need) {
      r.whole = true;
      break;
    }
  }
  return r;
}

// Marks in_set[j] (bit flags in `flags`, value `bit`) for the top c keys.
__device__ void warp_mark_top(const unsigned long long* keys, int n, int c, unsigned* hist,
                              uint8_t* flags, uint8_t bit) {
  const int lane = threadIdx.x & 31;
  if (c <= 0) return;
  if (c >= n) {
    for (int j = lane; j < n; j += 32) flags[j] |= bit;
    __syncwarp();
    return;
  }
  const TopSel t = warp_select_top(keys, n, c, hist);
  int taken = 0;  // equal keys taken so far, in index order
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool in = false, eq = false;
    if (j < n) {
      const unsigned long long km = keys[j] & t.mask;
      in = km > t.prefix;
      eq = km == t.prefix;
    }
    if (t.whole) {
      in = in || eq;
    } else {
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      const int rank = taken + __popc(eqb & ((1u << lane) - 1u));
      in = in || (eq && rank < t.need);
      taken += __popc(eqb);
    }
    if (in) flags[j] |= bit;
  }
  __syncwarp();
}

// Ascending list of the j < n with (flags[j] & bit) == want into out.
__device__ void warp_compact(const uint8_t* flags, int n, uint8_t bit, uint8_t want, int32_t* out) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const bool sel = j < n && ((flags[j] & bit) == want);
    const unsigned b = __ballot_sync(0xffffffffu, sel);
    if (sel) out[base + __popc(b & ((1u << lane) - 1u))] = j;
    base += __popc(b);
  }
}

// ---------------------------------------------------------------------------
// Both class boundaries of a three-way row: exact order statistics of the keys
// (score descending, lower block index first on equal scores).
// ---------------------------------------------------------------------------
constexpr int kClsBins = 512;  // histogram digits (9 bits per radix level)

__device__ __forceinline__ double order_key_value(unsigned long long k) {
  const unsigned long long b = (k & 0x8000000000000000ull) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double((long long)b);
}

// One level of the radix select over the keys of the interval [a, b] (as key - a,
// unsigned): 512 digits of (u - a) >> shift. Returns the digit holding the r-th
// largest of those keys (r >= 1, counting from the top) and the number of keys in
// the interval above that digit. hist: this warp's 512 counters.
struct Level {
  int digit;
  int above;   // keys of the interval in higher digits
  int count;   // keys in the digit
};

__device__ __forceinline__ Level radix_level(const unsigned long long* keys, int n, unsigned long long a,
                                             unsigned long long b, int shift, int r, unsigned* hist) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < kClsBins / 32; ++u) hist[lane + 32 * u] = 0u;
  __syncwarp();
  for (int j = lane; j < n; j += 32) {
    const unsigned long long kk = keys[j];
    if (kk >= a && kk <= b) atomicAdd(&hist[(unsigned)((kk - a) >> shift)], 1u);
  }
  __syncwarp();
  // lane l owns digits 511 - 16 l .. 496 - 16 l (descending)
  unsigned cnt[16], tot = 0;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    cnt[u] = hist[kClsBins - 1 - 16 * lane - u];
    tot += cnt[u];
  }
  unsigned incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)r);
  const int owner = __ffs(hit) - 1;  // r <= keys in the interval: some lane reaches it
  Level lv{0, 0, 0};
  if (lane == owner) {
    unsigned run = incl - tot;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (run + cnt[u] >= (unsigned)r) {
        lv.digit = kClsBins - 1 - 16 * lane - u;
        lv.above = (int)run;
        lv.count = (int)cnt[u];
        break;
      }
      run += cnt[u];
    }
  }
  lv.digit = __shfl_sync(0xffffffffu, lv.digit, owner);
  lv.above = __shfl_sync(0xffffffffu, lv.above, owner);
  lv.count = __shfl_sync(0xffffffffu, lv.count, owner);
  __syncwarp();
  return lv;
}

// The c-th element (1 <= c <= n) of the order "key descending, lower index first"
// of keys[0..n): returns its key and index. Exact: the interval holding it is
// narrowed one 9-bit digit at a time until it is a single key value, and among
// equal keys the (r)-th lowest index is taken.
__device__ void select_rank(const unsigned long long* keys, int n, int c, unsigned long long kmin,
                            unsigned long long kmax, unsigned* hist, unsigned long long* key_out, int* idx_out) {
  const int lane = threadIdx.x & 31;
  unsigned long long a = kmin, b = kmax;
  int r = c;
  while (a != b) {
    const unsigned long long span = b - a;
    const int bits = 64 - __clzll((long long)span);  // span < 2^bits
    const int shift = bits > 9 ? bits - 9 : 0;
    const Level lv = radix_level(keys, n, a, b, shift, r, hist);
    r -= lv.above;
    const unsigned long long lo = a + ((unsigned long long)lv.digit << shift);
    const unsigned long long hi_excl = shift >= 64 ? 0ull : ((unsigned long long)(lv.digit + 1) << shift);
    const unsigned long long hi = (hi_excl == 0ull || a + hi_excl - 1 < a || a + hi_excl - 1 > b) ? b : a + hi_excl - 1;
    a = lo;
    b = hi;
    if (shift == 0) break;  // one key value per digit
  }
  // a == b: the r-th lowest index among the keys equal to a
  int seen = 0, idx = -1;
  for (int j0 = 0; j0 < n && idx < 0; j0 += 32) {
    const int j = j0 + lane;
    const bool eq = j < n && keys[j] == a;
    const unsigned m = __ballot_sync(0xffffffffu, eq);
    const int cnt = __popc(m);
    if (seen + cnt >= r) {
      // the (r - seen)-th set bit of m
      unsigned mm = m;
      for (int q = 1; q < r - seen; ++q) mm &= mm - 1;
      idx = j0 + __ffs(mm) - 1;
    }
    seen += cnt;
  }
  *key_out = a;
  *idx_out = idx;
}

// Both class boundaries of one row in one pass. Digit 0 holds the filtered blocks
// (-inf), digits 1..511 split [min, max] of the finite scores linearly (a monotone
// map of the value, so the order of the digits is the order of the scores). The
// boundary digit of each boundary is found from the histogram; the keys in it are
// ranked exactly by comparing them with each other (lower block index first on
// equal keys). A digit with more than 32 keys falls back to select_rank.
struct Boundary {
  unsigned long long key;
  int idx;
};

__device__ void select_two(const unsigned long long* keys, int n, const int (&cnt)[2], unsigned long long kmin_f,
                           unsigned long long kmax_f, bool any_finite, unsigned long long kmin, unsigned long long kmax,
                           unsigned* hist, Boundary (&out)[2]) {
  const int lane = threadIdx.x & 31;
  const double smin = any_finite ? order_key_value(kmin_f) : 0.0, smax = any_finite ? order_key_value(kmax_f) : 0.0;
  double fac = smax > smin ? 510.0 / (smax - smin) : 0.0;
  if (!(fac < 1e300)) fac = 0.0;  // a subnormal range: one digit (its keys are then ranked exactly)
  auto digit = [&](unsigned long long kk) -> int {
    const double v = order_key_value(kk);
    if (v == -INFINITY) return 0;
    int d = 1 + (int)((v - smin) * fac);
    return d > kClsBins - 1 ? kClsBins - 1 : (d < 1 ? 1 : d);
  };
#pragma unroll
  for (int u = 0; u < kClsBins / 32; ++u) hist[lane + 32 * u] = 0u;
  __syncwarp();
  for (int j = lane; j < n; j += 32) atomicAdd(&hist[digit(keys[j])], 1u);
  __syncwarp();
  // lane l owns digits 511 - 16 l .. 496 - 16 l (descending)
  unsigned c16[16], tot = 0;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    c16[u] = hist[kClsBins - 1 - 16 * lane - u];
    tot += c16[u];
  }
  unsigned incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int bdig[2], need[2], bcnt[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const int r = cnt[b];
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)r);
    const int owner = __ffs(hit) - 1;
    int dg = 0, above = 0, inb = 0;
    if (lane == owner) {
      unsigned run = incl - tot;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (run + c16[u] >= (unsigned)r) {
          dg = kClsBins - 1 - 16 * lane - u;
          above = (int)run;
          inb = (int)c16[u];
          break;
        }
        run += c16[u];
      }
    }
    bdig[b] = __shfl_sync(0xffffffffu, dg, owner);
    need[b] = r - __shfl_sync(0xffffffffu, above, owner);
    bcnt[b] = __shfl_sync(0xffffffffu, inb, owner);
  }
  __syncwarp();
  // candidates of each boundary digit, ranked among themselves
  unsigned long long* ck = reinterpret_cast<unsigned long long*>(hist);  // 32 keys
  int* ci = reinterpret_cast<int*>(hist + 64);                           // 32 indices
#pragma unroll 1
  for (int b = 0; b < 2; ++b) {
    if (bcnt[b] > 32) {
      select_rank(keys, n, cnt[b], kmin, kmax, hist, &out[b].key, &out[b].idx);
      continue;
    }
    int base = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const bool is = j < n && digit(keys[j]) == bdig[b];
      const unsigned m = __ballot_sync(0xffffffffu, is);
      if (is) {
        const int pos = base + __popc(m & ((1u << lane) - 1u));
        ck[pos] = keys[j];
        ci[pos] = j;
      }
      base += __popc(m);
    }
    __syncwarp();
    const int c = bcnt[b];
    int rank = 1 << 30;
    unsigned long long mk = 0;
    int mi = -1;
    if (lane < c) {
      mk = ck[lane];
      mi = ci[lane];
      rank = 0;
      for (int t = 0; t < c; ++t) {
        const unsigned long long ok = ck[t];
        rank += (ok > mk || (ok == mk && ci[t] < mi)) ? 1 : 0;
      }
    }
    const unsigned win = __ballot_sync(0xffffffffu, rank == need[b] - 1);
    const int wl = win ? __ffs(win) - 1 : 0;
    out[b].key = __shfl_sync(0xffffffffu, mk, wl);
    out[b].idx = win ? __shfl_sync(0xffffffffu, mi, wl) : -1;
    __syncwarp();
  }
}

constexpr int kRouteWarps = 8;

// per warp of the classify kernel: the row's keys, then the histogram / candidates
__host__ __device__ inline size_t classify_warp_bytes(int nb) { return align_up((size_t)nb * 8, 16) + kClsBins * 4; }

static int route_rows_per_cta(int nb) {
  int r = (int)((96 * 1024) / classify_warp_bytes(nb));
  return r < 1 ? 1 : (r > kRouteWarps ? kRouteWarps : r);
}

static size_t route_smem(int nb, int rows) { return (size_t)rows * classify_warp_bytes(nb); }

// ---------------------------------------------------------------------------
// three-way classification: one warp per (b, h, query block i). The k_h-th and
// the (nb - k_l)-th block of the row's order are found exactly (select_two); a
// block is critical when it ranks at or before the first, negligible when it ranks
// after the second, marginal otherwise. Class = 2 critical, 1 marginal, 0 negligible.
// ---------------------------------------------------------------------------
__global__ void classify_kernel(const double* __restrict__ scores, int8_t* __restrict__ mask_out,
                                int32_t* __restrict__ crit, int32_t* __restrict__ neg,
                                __nv_bfloat16* __restrict__ mmask, int nb, int k_h, int k_l,
                                int nkb_pad, int nqb_pad, int rows, int n_rows, int linear_all,
                                const uint8_t* __restrict__ kflag, int H, int group, int* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * rows + w;  // over B*H*nqb_pad
  if (w >= rows || row >= n_rows) return;
  const int bh = row / nqb_pad, i = row % nqb_pad;
  if (i >= nb) {
    // rows past the last query block of the aggregation mask are zero
    if (mmask) {
      __nv_bfloat16* mrow = mmask + ((size_t)bh * nqb_pad + i) * nkb_pad;
      for (int j = lane; j < nkb_pad; j += 32) mrow[j] = __float2bfloat16(0.f);
    }
    return;
  }
  unsigned char* base = smem + (size_t)w * classify_warp_bytes(nb);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(base);
  unsigned* hist = reinterpret_cast<unsigned*>(base + align_up((size_t)nb * 8, 16));
  const double* srow = scores + ((size_t)bh * nb + i) * nb;
  // the score row lands in the key buffer with 16-byte copies, all in flight together
  // (rows start on 16 bytes when nb is even; otherwise element by element)
  {
    double* dst = reinterpret_cast<double*>(keys);
    if ((nb & 1) == 0) {
      for (int e = lane; e < nb / 2; e += 32) cp_async16(smem_u32(dst + 2 * e), srow + 2 * e, 16);
      cp_async_commit();
      cp_async_wait<0>();
    } else {
      for (int j = lane; j < nb; j += 32) dst[j] = srow[j];
    }
    __syncwarp();
  }
  // filtered key blocks (cos_filter) score -inf
  const uint8_t* kf = kflag ? kflag + ((size_t)(bh / H) * (H / group) + (bh % H) / group) * nb : nullptr;
  unsigned long long kmin = ~0ull, kmax = 0ull, fmin = ~0ull, fmax = 0ull;
  for (int j = lane; j < nb; j += 32) {
    const double v = kf && kf[j] ? -INFINITY : reinterpret_cast<const double*>(keys)[j];
    const unsigned long long kk = order_key(v);
    keys[j] = kk;
    kmin = kk < kmin ? kk : kmin;
    kmax = kk > kmax ? kk : kmax;
    if (v != -INFINITY) {
      fmin = kk < fmin ? kk : fmin;
      fmax = kk > fmax ? kk : fmax;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o), c = __shfl_xor_sync(0xffffffffu, kmax, o);
    kmin = a < kmin ? a : kmin;
    kmax = c > kmax ? c : kmax;
    a = __shfl_xor_sync(0xffffffffu, fmin, o);
    c = __shfl_xor_sync(0xffffffffu, fmax, o);
    fmin = a < fmin ? a : fmin;
    fmax = c > fmax ? c : fmax;
  }
  __syncwarp();
  // the k_h-th block (last critical) and the (nb - k_l)-th (last non-negligible)
  const bool c_some = k_h > 0, c_all = k_h >= nb;
  const bool n_some = nb - k_l > 0, n_all = k_l == 0;
  const int cnt2[2] = {c_some && !c_all ? k_h : 1, n_some && !n_all ? nb - k_l : 1};
  Boundary bd[2];
  select_two(keys, nb, cnt2, fmin, fmax, fmax >= fmin, kmin, kmax, hist, bd);
  const unsigned long long c_key = bd[0].key, n_key = bd[1].key;
  const int c_idx = (c_some && !c_all) ? bd[0].idx : -1, n_idx = (n_some && !n_all) ? bd[1].idx : -1;
  if ((c_some && !c_all && c_idx < 0) || (n_some && !n_all && n_idx < 0))
    if (lane == 0) report(status, SLA_ERR_DEVICE_CHECK, kDetailRouteSelect);
  const size_t rowoff = ((size_t)bh * nb + i) * nb;
  int nc_w = 0, nn_w = 0;
  int32_t* clist = crit && k_h > 0 ? crit + ((size_t)bh * nb + i) * k_h : nullptr;
  int32_t* nlist = neg && k_l > 0 ? neg + ((size_t)bh * nb + i) * k_l : nullptr;
  __nv_bfloat16* mrow = mmask ? mmask + ((size_t)bh * nqb_pad + i) * nkb_pad : nullptr;
  const int jend = mrow ? nkb_pad : nb;
  for (int j0 = 0; j0 < jend; j0 += 32) {
    const int j = j0 + lane;
    int cls = 0;
    if (j < nb) {
      const unsigned long long kk = keys[j];
      const bool is_c = c_all || (c_some && (kk > c_key || (kk == c_key && j <= c_idx)));
      const bool is_n = n_all || (n_some && (kk > n_key || (kk == n_key && j <= n_idx)));
      cls = is_c ? 2 : (is_n ? 1 : 0);
      if (mask_out) mask_out[rowoff + j] = (int8_t)cls;
    }
    // the aggregation mask: the marginal blocks, or every block with linear_all
    if (mrow && j < nkb_pad) mrow[j] = __float2bfloat16(j < nb && (linear_all || cls == 1) ? 1.f : 0.f);
    const unsigned bc = __ballot_sync(0xffffffffu, j < nb && cls == 2);
    const unsigned bn = __ballot_sync(0xffffffffu, j < nb && cls == 0);
    const unsigned below = (1u << lane) - 1u;
    if (clist && j < nb && cls == 2) {
      const int pos = nc_w + __popc(bc & below);
      if (pos < k_h) clist[pos] = j;
    }
    if (nlist && j < nb && cls == 0) {
      const int pos = nn_w + __popc(bn & below);
      if (pos < k_l) nlist[pos] = j;
    }
    nc_w += __popc(bc);
    nn_w += __popc(bn);
  }
  if (lane == 0 && ((clist && nc_w != k_h) || (nlist && nn_w != k_l)))
    report(status, SLA_ERR_DEVICE_CHECK, kDetailRouteSelect);
}

cudaError_t launch_classify(const Plan& p, const Args& a, bool write_mmask, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* sc = reinterpret_cast<const double*>(a.ws + p.off_scores);
  __nv_bfloat16* mm = write_mmask ? reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_mmask) : nullptr;
  const int rows = route_rows_per_cta(p.nkb);
  const size_t smem = route_smem(p.nkb, rows);
  cudaError_t e = cudaFuncSetAttribute(classify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // with the aggregation mask, rows nqb..nqb_pad (zero padding) get warps too
  const int per_head = write_mmask ? p.nqb_pad : p.nqb;
  const int n_rows = c.B * c.H * per_head;
  const int grid = (n_rows + rows - 1) / rows;
  classify_kernel<<<grid, rows * 32, smem, s>>>(sc, a.mask_out, a.crit, a.neg, mm, p.nkb, c.k_h,
                                                c.k_l, p.nkb_pad, per_head, rows, n_rows, c.linear_all,
                                                c.cos_filter ? reinterpret_cast<const uint8_t*>(a.ws + p.off_kflag)
                                                             : nullptr,
                                                c.H, p.group, a.status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// top-n selection: one warp per (b, KV head, query block i). Each of the
// group's heads takes a softmax of its pooled scores over the past blocks
// j < i (float64); the probabilities are summed and the top min(top_n, i)
// kept (same exact select as above). A head's score row is first copied into
// the warp's shared buffer with 16-byte loads, all in flight together; the
// max, the exponentials (one per element) and the sums then work from there.
// ---------------------------------------------------------------------------
// per warp: keys, row buffer (16-byte aligned), flags, histogram
__host__ __device__ inline size_t select_buf_off(int nb) { return align_up((size_t)nb * 8, 16); }
__host__ __device__ inline size_t select_warp_bytes(int nb) {
  return 2 * select_buf_off(nb) + align_up((size_t)nb, 16) + 1024;
}

__global__ void select_kernel(const double* __restrict__ scores, int8_t* __restrict__ mask_out,
                              int32_t* __restrict__ sel, int H, int group, int nb, int top_n,
                              int rows, int n_rows, const uint8_t* __restrict__ kflag) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * rows + w;  // over B*H_kv*nb
  if (w >= rows || row >= n_rows) return;
  const int bkv = row / nb, i = row % nb;
  const int Hkv = H / group;
  const int b = bkv / Hkv, hk = bkv % Hkv;
  unsigned char* base = smem + (size_t)w * select_warp_bytes(nb);
  double* prob = reinterpret_cast<double*>(base);  // becomes the keys
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(base);
  double* buf = reinterpret_cast<double*>(base + select_buf_off(nb));
  uint8_t* flags = base + 2 * select_buf_off(nb);
  unsigned* hist = reinterpret_cast<unsigned*>(base + 2 * select_buf_off(nb) + align_up((size_t)nb, 16));
  for (int j = lane; j < i; j += 32) {
    prob[j] = 0.0;
    flags[j] = 0;
  }
  __syncwarp();
  // score rows start on 16 bytes when nb is even: pairs, then the odd last one
  const int i2 = (nb & 1) ? 0 : (i & ~1);
  for (int g = 0; g < group && i > 0; ++g) {
    const double* srow = scores + (((size_t)b * H + hk * group + g) * nb + i) * nb;
#pragma unroll 4
    for (int j = 2 * lane; j < i2; j += 64)
      *reinterpret_cast<double2*>(buf + j) = *reinterpret_cast<const double2*>(srow + j);
#pragma unroll 4
    for (int j = i2 + lane; j < i; j += 32) buf[j] = srow[j];
    __syncwarp();
    if (kflag)  // filtered key blocks (cos_filter) score -inf
      for (int j = lane; j < i; j += 32)
        if (kflag[(size_t)bkv * nb + j]) buf[j] = -INFINITY;
    __syncwarp();
    double m = -INFINITY;
    for (int j = lane; j < i; j += 32) m = fmax(m, buf[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (m == -INFINITY) continue;  // every candidate filtered: this head adds 0
    double sum = 0.0;
    for (int j = lane; j < i; j += 32) {
      const double e = exp(buf[j] - m);
      buf[j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const double inv = 1.0 / sum;
    for (int j = lane; j < i; j += 32) prob[j] += buf[j] * inv;
    __syncwarp();
  }
  for (int j = lane; j < i; j += 32) keys[j] = order_key(prob[j]);
  __syncwarp();
  const int n = i < top_n ? i : top_n;
  warp_mark_top(keys, i, n, hist, flags, 1);
  const size_t rowid = (size_t)bkv * nb + i;
  int32_t* lst = sel + rowid * top_n;
  if (top_n > 0) {
    warp_compact(flags, i, 1, 1, lst);
    for (int u = n + lane; u < top_n; u += 32) lst[u] = -1;
  }
  if (mask_out)
    for (int j = lane; j < nb; j += 32) mask_out[rowid * nb + j] = (j < i && (flags[j] & 1)) ? 2 : 0;
}

cudaError_t launch_select(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const double* sc = reinterpret_cast<const double*>(a.ws + p.off_scores);
  const size_t per = select_warp_bytes(p.nkb);
  int rows = (int)((96 * 1024) / per);
  rows = rows < 1 ? 1 : (rows > kRouteWarps ? kRouteWarps : rows);
  const size_t smem = (size_t)rows * per;
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_rows = c.B * c.H_kv * p.nqb;
  const int grid = (n_rows + rows - 1) / rows;
  select_kernel<<<grid, rows * 32, smem, s>>>(
      sc, a.mask_out, a.crit, c.H, p.group, p.nkb, c.top_n, rows, n_rows,
      c.cos_filter ? reinterpret_cast<const uint8_t*>(a.ws + p.off_kflag) : nullptr);
  return cudaGetLastError();
}

}  // namespace sla
