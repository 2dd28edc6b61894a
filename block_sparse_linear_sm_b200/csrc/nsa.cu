// NSA's three parallel branches (top-n mode with nsa_branches).
//
// Sparse attention survey, section 2 (NSA): a compressed branch over coarse blocks
// of 32 tokens at stride 16 (global context at low cost), the selected branch (the
// top blocks of 64 tokens) and the sliding window, in parallel. The pages give no
// compression function and no gate form; here a compressed key (value) is the mean
// of its block's tokens, each branch is its own softmax, and the branches are
// summed with per-head gates g_b = sigmoid(q . w_g[h][b]) (g_b = 1 without gates).
// The three attentions run in the sparse flash kernel (flash_tc.cu): the compressed
// branch over the compressed keys, every tile up to the causal limit c * stride +
// length - 1 <= t; the window branch's epilogue writes the gated sum. This file holds
// the compression, HBM-bound, one warp per compressed row, and the first step of the
// backward pass of the three branches (nsa_prep_kernel).
#include "common.cuh"

namespace sla {

// kc / vc row c of KV head bkv = mean of k / v rows c*stride .. c*stride + len - 1 (all
// valid); rows n_cmp .. ncmp_pad - 1 are zero. Each lane owns d / 32 features.
template <int D>
__global__ void compress_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc, int64_t rows,
                                int N, int n_cmp, int ncmp_pad, int len, int stride) {
  constexpr int E = D / 32;  // features per lane: 4 (d = 128) or 2 (d = 64)
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float inv = 1.f / (float)len;
  for (int64_t r = w0; r < rows; r += nw) {
    const int64_t bkv = r / ncmp_pad;
    const int c = (int)(r % ncmp_pad);
    for (int which = 0; which < 2; ++which) {
      const __nv_bfloat16* src = (which == 0 ? k : v) + (size_t)bkv * N * D + lane * E;
      float acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      if (c < n_cmp)
        for (int t = c * stride; t < c * stride + len; ++t) {
          const __nv_bfloat16* x = src + (size_t)t * D;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] += __bfloat162float(x[e]);
        }
      __nv_bfloat16* dst = (which == 0 ? kc : vc) + (size_t)r * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) dst[e] = __float2bfloat16(acc[e] * inv);
    }
  }
}

cudaError_t launch_compress(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const int64_t rows = (int64_t)c.B * c.H_kv * p.ncmp_pad;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  auto* kc = reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_kc);
  auto* vc = reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_vc);
  if (c.d == 128)
    compress_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(a.k, a.v, kc, vc, rows, c.N, p.n_cmp, p.ncmp_pad,
                                                          c.cmp_block, c.cmp_stride);
  else
    compress_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(a.k, a.v, kc, vc, rows, c.N, p.n_cmp, p.ncmp_pad,
                                                         c.cmp_block, c.cmp_stride);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Backward pass, per row t of head h (loss L = sum(O * dO), O = sum_b g_b o_b):
//   e_b = dO_t . o_b,t; the branch's attention gradient is that of softmax attention
//   with output gradient g_b dO_t, whose D value is g_b e_b. The flash kernels recompute
//   P with lse_b - log2 g_b (P scaled by g_b) and take D = e_b, which gives the same dS,
//   dK, dV and dQ; dlogit_b = e_b g_b (1 - g_b) (sigmoid gate, g_b = 1 without gates);
//   dq_t += sum_b dlogit_b w_g[h][b] (in the dQ kernel), dw_g[h][b] += sum_t dlogit_b q_t.
// One CTA per 256 rows of a head, a warp per row, lane = D / 32 features; the dw_g
// partials of the CTA are summed in shared memory and added with one atomic per element.
// Padding rows: lse = +inf, e = dlogit = 0.
// ---------------------------------------------------------------------------
constexpr int kPrepRows = 256, kPrepWarps = 8;

template <int D>
__global__ void __launch_bounds__(kPrepWarps * 32)
    nsa_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                    const __nv_bfloat16* __restrict__ oc, const __nv_bfloat16* __restrict__ os,
                    const __nv_bfloat16* __restrict__ ow, const __nv_bfloat16* __restrict__ w_g3,
                    const float* __restrict__ lse_in, float* __restrict__ lse_out, float* __restrict__ delta,
                    float* __restrict__ dlogit, float* __restrict__ dw_g, int H, int N, int n_valid,
                    size_t bstride) {
  constexpr int E = D / 32;
  __shared__ float red[kPrepWarps][3][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunks = (N + kPrepRows - 1) / kPrepRows;
  const int bh = blockIdx.x / chunks, t0 = (blockIdx.x % chunks) * kPrepRows;
  const int h = bh % H;
  float wg[3][E], acc[3][E];
#pragma unroll
  for (int b = 0; b < 3; ++b)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      wg[b][e] = w_g3 ? __bfloat162float(w_g3[((size_t)h * 3 + b) * D + lane * E + e]) : 0.f;
      acc[b][e] = 0.f;
    }
  for (int t = t0 + warp; t < t0 + kPrepRows && t < N; t += kPrepWarps) {
    const size_t row = (size_t)bh * N + t;
    float ev[3] = {0.f, 0.f, 0.f}, dot[3] = {0.f, 0.f, 0.f}, qv[E];
    const bool valid = t < n_valid;
    if (valid) {
      const __nv_bfloat16* src[3] = {oc + row * D, os + row * D, ow + row * D};
      const __nv_bfloat16* g = dout + row * D + lane * E;
      const __nv_bfloat16* qq = q + row * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float go = __bfloat162float(g[e]);
        qv[e] = __bfloat162float(qq[e]);
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          ev[b] = fmaf(go, __bfloat162float(src[b][lane * E + e]), ev[b]);
          dot[b] = fmaf(qv[e], wg[b][e], dot[b]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          ev[b] += __shfl_xor_sync(0xffffffffu, ev[b], o);
          dot[b] += __shfl_xor_sync(0xffffffffu, dot[b], o);
        }
    }
#pragma unroll
    for (int b = 0; b < 3; ++b) {
      float lse = INFINITY, dl = 0.f;
      if (valid) {
        lse = lse_in[b * bstride + row];
        if (w_g3) {
          const float gb = 1.f / (1.f + __expf(-dot[b]));
          lse -= log2f(gb);  // +inf stays +inf; gb = 0 gives +inf (P = 0)
          dl = ev[b] * gb * (1.f - gb);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[b][e] = fmaf(dl, qv[e], acc[b][e]);
        }
      }
      if (lane == 0) {
        lse_out[b * bstride + row] = lse;
        delta[b * bstride + row] = valid ? ev[b] : 0.f;
        if (dlogit) dlogit[b * bstride + row] = dl;
      }
    }
  }
  if (!w_g3) return;
#pragma unroll
  for (int b = 0; b < 3; ++b)
#pragma unroll
    for (int e = 0; e < E; ++e) red[warp][b][lane * E + e] = acc[b][e];
  __syncthreads();
  for (int x = threadIdx.x; x < 3 * D; x += blockDim.x) {
    const int b = x / D, col = x % D;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kPrepWarps; ++w) sum += red[w][b][col];
    atomicAdd(dw_g + ((size_t)h * 3 + b) * D + col, sum);
  }
}

cudaError_t launch_nsa_prep(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const int chunks = (c.N + kPrepRows - 1) / kPrepRows;
  const unsigned grid = (unsigned)(c.B * c.H * chunks);
  const size_t bstride = (size_t)c.B * c.H * c.N;
  const auto* oc = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_oc);
  const auto* os = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_os);
  const auto* ow = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_ow);
  const auto* lse_in = reinterpret_cast<const float*>(a.ws + p.off_lse);
  auto* lse_out = reinterpret_cast<float*>(a.bws + bp.off_lse3);
  auto* delta = reinterpret_cast<float*>(a.bws + bp.off_delta);
  float* dlogit = c.has_gate ? reinterpret_cast<float*>(a.bws + bp.off_dlogit) : nullptr;
  const __nv_bfloat16* wg = c.has_gate ? a.w_g : nullptr;
  if (c.d == 128)
    nsa_prep_kernel<128><<<grid, kPrepWarps * 32, 0, s>>>(a.q, a.dout, oc, os, ow, wg, lse_in, lse_out, delta, dlogit,
                                                          a.dw_g, c.H, c.N, c.N_valid, bstride);
  else
    nsa_prep_kernel<64><<<grid, kPrepWarps * 32, 0, s>>>(a.q, a.dout, oc, os, ow, wg, lse_in, lse_out, delta, dlogit,
                                                         a.dw_g, c.H, c.N, c.N_valid, bstride);
  return cudaGetLastError();
}

}  // namespace sla
