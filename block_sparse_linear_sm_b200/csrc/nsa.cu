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
// the compression, HBM-bound, one warp per compressed row.
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

}  // namespace sla
