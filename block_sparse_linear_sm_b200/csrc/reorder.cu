// Token reordering along a 3-D Hilbert curve (2025 review, section 11,
// SpargeAttn: ordering tokens along a Hilbert curve raises the similarity of
// the tokens that share a block, which sharpens the block-level prediction).
//
// sla_hilbert_order (host): the curve index of every (t, h, w) grid point on the
// smallest power-of-two cube holding the grid, by Skilling's axes-to-transpose
// method ("Programming the Hilbert curve", AIP Conf. Proc. 707, 2004), then the
// raster indices sorted by it. The order depends only on the grid, so a caller
// computes it once per video shape and keeps it on the device.
// sla_permute_tokens (device): y[row, n'] = x[row, order[n']] (inverse: the
// scatter back), 16 bytes per thread, coalesced on the contiguous side.
#include <stdint.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "common.cuh"

namespace sla {

// Curve index of (x, y, z) on the cube of side 2^bits.
static uint64_t hilbert_key3(uint32_t x, uint32_t y, uint32_t z, int bits) {
  uint32_t a[3] = {x, y, z};
  const uint32_t top = 1u << (bits - 1);
  // undo the excess work, from the top level down: invert or exchange low bits
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (a[i] & q) {
        a[0] ^= low;
      } else {
        const uint32_t swap = (a[0] ^ a[i]) & low;
        a[0] ^= swap;
        a[i] ^= swap;
      }
    }
  }
  // Gray-encode across the axes
  for (int i = 1; i < 3; ++i) a[i] ^= a[i - 1];
  uint32_t flip = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (a[2] & q) flip ^= q - 1;
  for (int i = 0; i < 3; ++i) a[i] ^= flip;
  // the transposed index, read level by level, first axis most significant
  uint64_t key = 0;
  for (int b = bits - 1; b >= 0; --b)
    for (int i = 0; i < 3; ++i) key = (key << 1) | ((a[i] >> b) & 1u);
  return key;
}

__global__ void permute_tokens_kernel(const uint4* __restrict__ x, uint4* __restrict__ y,
                                      const int32_t* __restrict__ order, int n_order, int n_tok,
                                      int chunks, long long total, int inverse) {
  // one thread per 16-byte chunk of one token row of one head row
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % chunks);
    const long long tokrow = e / chunks;  // head row * n_tok + token
    const int n = (int)(tokrow % n_tok);
    const long long base = tokrow - n;
    int src = n, dst = n;
    if (n < n_order) {
      const int o = order[n];
      if (o < 0 || o >= n_order) continue;  // not a permutation entry: nothing is read or written
      if (inverse) dst = o;
      else src = o;
    }
    y[(base + dst) * chunks + c] = x[(base + src) * chunks + c];
  }
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_hilbert_order(int32_t t, int32_t h, int32_t w, int32_t* order) {
  if (t < 1 || h < 1 || w < 1 || !order) return SLA_ERR_INVALID_ARG;
  const int64_t n = (int64_t)t * h * w;
  if (n > ((int64_t)1 << 30)) return SLA_ERR_INVALID_ARG;
  const int32_t side = std::max(t, std::max(h, w));
  int bits = 1;
  while ((1 << bits) < side) ++bits;
  std::vector<uint64_t> key((size_t)n);
  for (int32_t a = 0; a < t; ++a)
    for (int32_t b = 0; b < h; ++b)
      for (int32_t c = 0; c < w; ++c)
        key[((size_t)a * h + b) * w + c] = hilbert_key3((uint32_t)a, (uint32_t)b, (uint32_t)c, bits);
  std::vector<int32_t> idx((size_t)n);
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t i, int32_t j) { return key[i] < key[j]; });
  std::copy(idx.begin(), idx.end(), order);
  return SLA_OK;
}

extern "C" sla_status sla_permute_tokens(const void* x, void* y, const int32_t* order, int32_t n_order,
                                         int32_t rows, int32_t n_tok, int32_t d, int32_t inverse,
                                         void* stream) {
  if (!x || !y || x == y || !order || rows < 1 || n_tok < 1 || n_order < 0 || n_order > n_tok)
    return SLA_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0) return SLA_ERR_INVALID_ARG;
  if (((uintptr_t)x % 16) || ((uintptr_t)y % 16) || ((uintptr_t)order % 4)) return SLA_ERR_INVALID_ARG;
  const int chunks = d / 8;  // 16-byte chunks of a bf16 row
  const long long total = (long long)rows * n_tok * chunks;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148LL * 32) blocks = 148LL * 32;  // grid-stride beyond 32 resident blocks per SM
  permute_tokens_kernel<<<(int)blocks, threads, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(y), order, n_order, n_tok, chunks, total,
      inverse);
  return cudaGetLastError() == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}
