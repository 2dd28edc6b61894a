// Epilogue of the three-way layer: apply the aggregated linear state, gate and
// add the sparse branch.
//
//   O[t] = O_s[t] + g_t * (phi(q_t) S'_i) / (phi(q_t) . Z_i),  g_t = sigmoid(q_t . w_g[h])
//
// SLA analysis page (arXiv 2509.24006), Proj paragraph: O = O^s + Proj(O^l);
// SALAD summary page, method details: an input-dependent gate balances the
// sparse and linear branches. S'_i already carries the projection
// (S'_i = sum_j phi(K_j)^T V_j W_p, folded in by the state kernel), so the
// projection costs no separate product here. Without a gate g = 1.
//
// One CTA per (b, h, query block): 4 warps of 16 rows. phi(q) (bf16) and S'_i
// (bf16) and O_s are staged in shared memory with cp.async (all loads in flight
// together); the product runs on mma.sync with fp32 accumulation; O is formed
// in the O_s tile and written with 16-byte stores. About 65 KB of shared
// memory, three CTAs per SM.
#include "common.cuh"

namespace sla {

struct EpiParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* os;   // [B*H][N][D] sparse branch
  const __nv_bfloat16* ss;   // [B*H][nqb][D*D] S'_i
  const float* zs;           // [B*H][nqb][D]   Z_i
  const __nv_bfloat16* w_g;  // [H][D] or null
  __nv_bfloat16* out;
  int H, N, n_valid, nb;
};

template <int D>
__global__ void __launch_bounds__(128) epilogue_kernel(EpiParams prm) {
  constexpr int RB = D * 2, CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* fq_s = smem;                      // [64][D]  q, then phi(q)
  unsigned char* s_s = fq_s + kBlock * RB;         // [D][D]   S'_i
  unsigned char* o_s = s_s + D * RB;               // [64][D]  O_s, then O
  float* z_s = reinterpret_cast<float*>(o_s + kBlock * RB);  // [D]
  float* den_s = z_s + D;                               // [64]
  float* g_s = den_s + kBlock;                          // [64]

  const int i = blockIdx.x, bh = blockIdx.y;
  const int h = bh % prm.H;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nvq = min(kBlock, prm.n_valid - i * kBlock);
  const __nv_bfloat16* qg = prm.q + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
  const __nv_bfloat16* sg = prm.ss + ((size_t)bh * prm.nb + i) * D * D;
  const float* zg = prm.zs + ((size_t)bh * prm.nb + i) * D;
  const uint32_t fq_b = smem_u32(fq_s), s_b = smem_u32(s_s), z_b = smem_u32(z_s), o_b = smem_u32(o_s);
  const __nv_bfloat16* osg = prm.os + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;

  // all loads in flight at once: S'_i, the query rows (padding rows zero), O_s, Z_i
  for (int e = tid; e < D * CH; e += 128) {
    const int r = e / CH, ch = e % CH;
    cp_async16(s_b + swz(r, ch, RB), sg + (size_t)r * D + ch * 8, 16);
  }
  for (int e = tid; e < kBlock * CH; e += 128) {
    const int t = e / CH, ch = e % CH;
    const int bytes = t < nvq ? 16 : 0;
    cp_async16(fq_b + swz(t, ch, RB), qg + (bytes ? (size_t)t * D + ch * 8 : 0), bytes);
  }
  for (int e = tid; e < kBlock * CH; e += 128) {
    const int t = e / CH, ch = e % CH;
    cp_async16(o_b + swz(t, ch, RB), osg + (size_t)t * D + ch * 8, 16);
  }
  for (int e = tid; e < D / 4; e += 128) cp_async16(z_b + e * 16, zg + e * 4, 16);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // gate from the raw query rows (2 threads per row)
  {
    const int r = tid >> 1, half = tid & 1;
    float acc = 0.f;
    if (prm.w_g) {
      const __nv_bfloat16* wg = prm.w_g + (size_t)h * D;
      for (int c8 = half * (CH / 2); c8 < (half + 1) * (CH / 2); ++c8) {
        const uint4 u = *reinterpret_cast<const uint4*>(fq_s + swz(r, c8, RB));
        const uint4 g = *reinterpret_cast<const uint4*>(wg + c8 * 8);
        const uint32_t* uu = reinterpret_cast<const uint32_t*>(&u);
        const uint32_t* gg = reinterpret_cast<const uint32_t*>(&g);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 a = unpack_bf16(uu[x]), b = unpack_bf16(gg[x]);
          acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
        }
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) g_s[r] = prm.w_g ? 1.f / (1.f + __expf(-acc)) : 1.f;
  }
  __syncthreads();
  // phi in place, and the denominators phi(q) . Z_i from the same bf16 values
  {
    const int r = tid >> 1, half = tid & 1;
    float acc = 0.f;
    for (int c8 = half * (CH / 2); c8 < (half + 1) * (CH / 2); ++c8) {
      uint4 u = *reinterpret_cast<const uint4*>(fq_s + swz(r, c8, RB));
      uint32_t* uu = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float2 a = unpack_bf16(uu[x]);
        uu[x] = pack_bf16(phi(a.x), phi(a.y));
        const float2 f = unpack_bf16(uu[x]);
        acc = fmaf(f.x, z_s[c8 * 8 + 2 * x], fmaf(f.y, z_s[c8 * 8 + 2 * x + 1], acc));
      }
      *reinterpret_cast<uint4*>(fq_s + swz(r, c8, RB)) = u;
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) den_s[r] = acc;
  }
  __syncthreads();

  float num[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) num[n][0] = num[n][1] = num[n][2] = num[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[4];
    ldsm_x4(lds_a(fq_b, 16 * w, 2 * ks, RB, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n2 = 0; n2 < D / 16; ++n2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(lds_b_kn(s_b, ks * 16, 2 * n2, RB, lane), b0, b1, b2, b3);
      mma_bf16(num[2 * n2], a, b0, b1);
      mma_bf16(num[2 * n2 + 1], a, b2, b3);
    }
  }
  const int row0 = 16 * w + (lane >> 2);
  const float d0 = den_s[row0], d1 = den_s[row0 + 8];
  const float c0 = d0 > 0.f ? g_s[row0] / d0 : 0.f, c1 = d1 > 0.f ? g_s[row0 + 8] / d1 : 0.f;
  const bool v0 = row0 < nvq, v1 = row0 + 8 < nvq;
  // O = O_s + c * num in place in the O_s tile (each warp owns its 16 rows) ...
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * (lane & 3);
    uint32_t* p0 = reinterpret_cast<uint32_t*>(o_s + swz(row0, col >> 3, RB) + (col & 7) * 2);
    uint32_t* p1 = reinterpret_cast<uint32_t*>(o_s + swz(row0 + 8, col >> 3, RB) + (col & 7) * 2);
    const float2 s0 = unpack_bf16(*p0), s1 = unpack_bf16(*p1);
    *p0 = v0 ? pack_bf16(s0.x + c0 * num[n][0], s0.y + c0 * num[n][1]) : 0u;
    *p1 = v1 ? pack_bf16(s1.x + c1 * num[n][2], s1.y + c1 * num[n][3]) : 0u;
  }
  __syncwarp();
  // ... then 16-byte coalesced stores of the warp's rows
  __nv_bfloat16* og = prm.out + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
  for (int e = lane; e < 16 * CH; e += 32) {
    const int t = 16 * w + e / CH, ch = e % CH;
    *reinterpret_cast<uint4*>(og + (size_t)t * D + ch * 8) =
        *reinterpret_cast<const uint4*>(o_s + swz(t, ch, RB));
  }
}

template <int D>
static cudaError_t launch_epi_t(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  EpiParams prm;
  prm.q = a.q;
  prm.os = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_os);
  prm.ss = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_ss);
  prm.zs = reinterpret_cast<const float*>(a.ws + p.off_zs);
  prm.w_g = c.has_gate ? a.w_g : nullptr;
  prm.out = a.out;
  prm.H = c.H;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = p.nqb;
  const int smem = 2 * kBlock * D * 2 + D * D * 2 + (D + 2 * kBlock) * 4;
  cudaError_t e = cudaFuncSetAttribute(epilogue_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nqb, c.B * c.H);
  epilogue_kernel<D><<<grid, 128, smem, s>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_epilogue(const Plan& p, const Args& a, cudaStream_t s) {
  return p.c.d == 128 ? launch_epi_t<128>(p, a, s) : launch_epi_t<64>(p, a, s);
}

}  // namespace sla
