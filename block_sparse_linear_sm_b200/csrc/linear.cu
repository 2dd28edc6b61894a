// Linear branch of the layer: per-key-block states and their aggregation over
// each query block's marginal blocks.
//
// SLA analysis page (arXiv 2509.24006), comparison table and core-innovation
// paragraph: marginal blocks go through linear attention at O(N d^2). With
// phi = elu + 1 the branch factorises per key block j into the d x d state
// h_j = phi(K_j)^T V_j and the normaliser z_j = sum_t phi(k_t); query block i
// then needs S_i = sum_{j marginal} h_j and Z_i = sum_{j marginal} z_j.
//
// Layout: Hs[bkv][j][0 : d*d] = h_j row-major (times W_p when the layer has a
// projection: h'_j = phi(K_j)^T V_j W_p), Hs[bkv][j][d*d : d*d+d] = z_j,
// zero up to dd (a multiple of 128), rows j in [nkb, nkb_pad) zero; bf16.
// The aggregation over each query block's marginal blocks is a tcgen05 GEMM
// (aggregate_tc.cu).
#include "common.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// state kernel: one CTA per (b, kv head, key block); D/16 warps.
// With a projection, W_p is folded into the state: O_l W_p =
// phi(q) sum_j phi(K_j)^T (V_j W_p) / den, so the block first forms
// T_j = V_j W_p (warp w owns token rows 16(w%4).. of T, column half w/4), then
// h'_j = phi(K_j)^T T_j (warp w owns rows 16w..16w+15 of h'_j).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D * 2) state_kernel(const __nv_bfloat16* __restrict__ k,
                                                      const __nv_bfloat16* __restrict__ v,
                                                      const __nv_bfloat16* __restrict__ w_p,
                                                      __nv_bfloat16* __restrict__ hs, int N,
                                                      int n_valid, int nkb, int dd) {
  constexpr int RB = D * 2;  // bytes per smem row
  constexpr int CH = D / 8;  // 16-byte chunks per row
  constexpr int NW = D / 16; // warps
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* fk_s = smem;                    // [64][D]  phi(K)
  unsigned char* v_s = fk_s + kBlock * RB;       // [64][D]  V, then T = V W_p
  unsigned char* w_s = v_s + kBlock * RB;        // [D][D]   W_p (only with a projection)
  const int j = blockIdx.x;
  const int bkv = blockIdx.y;
  __nv_bfloat16* row = hs + ((size_t)bkv * gridDim.x + j) * dd;
  if (j >= nkb) {
    for (int e = threadIdx.x; e < dd / 8; e += blockDim.x)
      reinterpret_cast<uint4*>(row)[e] = make_uint4(0, 0, 0, 0);
    return;
  }
  int nv = n_valid - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  const __nv_bfloat16* kb = k + ((size_t)bkv * N + (size_t)j * kBlock) * D;
  const __nv_bfloat16* vb = v + ((size_t)bkv * N + (size_t)j * kBlock) * D;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t fk_base = smem_u32(fk_s), v_base = smem_u32(v_s), w_base = smem_u32(w_s);
  if (w_p) {
    for (int e = threadIdx.x; e < D * CH; e += blockDim.x) {
      const int r = e / CH, ch = e % CH;
      cp_async16(w_base + swz(r, ch, RB), w_p + (size_t)r * D + ch * 8, 16);
    }
  }
  for (int e = threadIdx.x; e < kBlock * CH; e += blockDim.x) {
    const int t = e / CH, ch = e % CH;
    const int bytes = t < nv ? 16 : 0;
    cp_async16(v_base + swz(t, ch, RB), vb + (bytes ? (size_t)t * D + ch * 8 : 0), bytes);
  }
  cp_async_commit();
  for (int e = threadIdx.x; e < kBlock * CH; e += blockDim.x) {
    const int t = e / CH, ch = e % CH;
    uint4 kk = make_uint4(0, 0, 0, 0);
    if (t < nv) {
      kk = *reinterpret_cast<const uint4*>(kb + (size_t)t * D + ch * 8);
      uint32_t* wv = reinterpret_cast<uint32_t*>(&kk);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float2 f = unpack_bf16(wv[u]);
        wv[u] = pack_bf16(phi(f.x), phi(f.y));
      }
    }
    *reinterpret_cast<uint4*>(fk_s + swz(t, ch, RB)) = kk;
  }
  cp_async_wait<0>();
  __syncthreads();
  // z_j from the same bf16-rounded features the MMA uses
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float z = 0.f;
    for (int t = 0; t < nv; ++t) {
      const __nv_bfloat16* p =
          reinterpret_cast<const __nv_bfloat16*>(fk_s + swz(t, c >> 3, RB)) + (c & 7);
      z += __bfloat162float(*p);
    }
    row[D * D + c] = __float2bfloat16(z);
  }
  for (int e = D * D + D + threadIdx.x; e < dd; e += blockDim.x) row[e] = __float2bfloat16(0.f);

  if (w_p) {
    // T = V W_p: warp w -> token rows 16*(w % 4) .., columns [half*D/2, (half+1)*D/2)
    constexpr int HALVES = NW / 4;  // 2 for D=128, 1 for D=64
    constexpr int NC = D / HALVES;  // columns per warp
    const int mt = w & 3, half = w >> 2;
    float t_acc[NC / 8][4];
#pragma unroll
    for (int n = 0; n < NC / 8; ++n) t_acc[n][0] = t_acc[n][1] = t_acc[n][2] = t_acc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(lds_a(v_base, mt * 16, 2 * ks, RB, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int n2 = 0; n2 < NC / 16; ++n2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(lds_b_kn(w_base, ks * 16, (half * NC) / 8 + 2 * n2, RB, lane), b0, b1, b2, b3);
        mma_bf16(t_acc[2 * n2], a, b0, b1);
        mma_bf16(t_acc[2 * n2 + 1], a, b2, b3);
      }
    }
    __syncthreads();  // every warp has read V: T may overwrite it
    const int r0 = mt * 16 + (lane >> 2);
#pragma unroll
    for (int n = 0; n < NC / 8; ++n) {
      const int col = half * NC + n * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(v_s + swz(r0, col >> 3, RB) + (col & 7) * 2) =
          pack_bf16(t_acc[n][0], t_acc[n][1]);
      *reinterpret_cast<uint32_t*>(v_s + swz(r0 + 8, col >> 3, RB) + (col & 7) * 2) =
          pack_bf16(t_acc[n][2], t_acc[n][3]);
    }
    __syncthreads();
  }

  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < kBlock / 16; ++ks) {
    uint32_t a[4];
    ldsm_x4_t(lds_a_km(fk_base, ks * 16, 2 * w, RB, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n2 = 0; n2 < D / 16; ++n2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(lds_b_kn(v_base, ks * 16, 2 * n2, RB, lane), b0, b1, b2, b3);
      mma_bf16(acc[2 * n2], a, b0, b1);
      mma_bf16(acc[2 * n2 + 1], a, b2, b3);
    }
  }
  const int r0 = 16 * w + (lane >> 2);
  const int cc = 2 * (lane & 3);
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    *reinterpret_cast<uint32_t*>(row + (size_t)r0 * D + n * 8 + cc) = pack_bf16(acc[n][0], acc[n][1]);
    *reinterpret_cast<uint32_t*>(row + (size_t)(r0 + 8) * D + n * 8 + cc) =
        pack_bf16(acc[n][2], acc[n][3]);
  }
}

cudaError_t launch_state(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_hs);
  const __nv_bfloat16* wp = c.has_proj ? a.w_p : nullptr;
  dim3 grid(p.nkb_pad, c.B * c.H_kv);
  if (c.d == 128) {
    const int smem = 2 * kBlock * 256 + (wp ? 128 * 256 : 0);
    cudaError_t e = cudaFuncSetAttribute(state_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    state_kernel<128><<<grid, 256, smem, s>>>(a.k, a.v, wp, hs, c.N, c.N_valid, p.nkb, p.dd);
  } else {
    const int smem = 2 * kBlock * 128 + (wp ? 64 * 128 : 0);
    state_kernel<64><<<grid, 128, smem, s>>>(a.k, a.v, wp, hs, c.N, c.N_valid, p.nkb, p.dd);
  }
  return cudaGetLastError();
}

}  // namespace sla
