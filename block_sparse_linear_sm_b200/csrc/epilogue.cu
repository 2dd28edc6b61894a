// Epilogue of the three-way layer: apply the aggregated linear state, project,
// gate and add the sparse branch.
//
//   O_l[t] = phi(q_t) S_i / (phi(q_t) . Z_i)          (0 when row i has no marginal block)
//   O[t]   = O_s[t] + g_t * (O_l[t] W_p),  g_t = sigmoid(q_t . w_g[h])
//
// SLA analysis page (arXiv 2509.24006), Proj paragraph: O = O^s + Proj(O^l);
// SALAD summary page, method details: an input-dependent gate balances the
// sparse and linear branches. Without projection W_p = I, without gate g = 1.
//
// One CTA per (b, h, query block), 4 warps of 16 rows. phi(q), S_i and W_p are
// staged in shared memory as bf16; both products run on mma.sync with fp32
// accumulation.
#include "common.cuh"

namespace sla {

struct EpiParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* os;   // [B*H][N][D] sparse branch
  const float* ss;           // [B*H][nqb][dd]: S_i (D*D) then Z_i (D)
  const __nv_bfloat16* w_p;  // [D][D] or null
  const __nv_bfloat16* w_g;  // [H][D] or null
  __nv_bfloat16* out;
  int H, N, n_valid, nb, dd;
  int has_marginal;
};

template <int D>
__global__ void __launch_bounds__(128) epilogue_kernel(EpiParams prm) {
  constexpr int RB = D * 2, CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* fq_s = smem;                      // [64][D]
  unsigned char* s_s = fq_s + kBlock * RB;         // [D][D]
  unsigned char* w_s = s_s + D * RB;               // [D][D]
  unsigned char* ol_s = w_s + D * RB;              // [64][D]
  float* z_s = reinterpret_cast<float*>(ol_s + kBlock * RB);  // [D]
  float* den_s = z_s + D;                                     // [64]
  float* g_s = den_s + kBlock;                                // [64]

  const int i = blockIdx.x, bh = blockIdx.y;
  const int h = bh % prm.H;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nvq = min(kBlock, prm.n_valid - i * kBlock);
  const __nv_bfloat16* qg = prm.q + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
  const bool use_lin = prm.has_marginal != 0;
  const bool proj = prm.w_p != nullptr;

  if (use_lin) {
    // phi(q) rows as bf16
    for (int e = tid; e < kBlock * CH; e += 128) {
      const int t = e / CH, ch = e % CH;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (t < nvq) {
        u = *reinterpret_cast<const uint4*>(qg + (size_t)t * D + ch * 8);
        uint32_t* wv = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float2 f = unpack_bf16(wv[x]);
          wv[x] = pack_bf16(phi(f.x), phi(f.y));
        }
      }
      *reinterpret_cast<uint4*>(fq_s + swz(t, ch, RB)) = u;
    }
    // S_i (fp32 -> bf16) and Z_i
    const float* sg = prm.ss + ((size_t)bh * prm.nb + i) * prm.dd;
    for (int e = tid; e < D * CH; e += 128) {
      const int r = e / CH, ch = e % CH;
      const float4 a = *reinterpret_cast<const float4*>(sg + (size_t)r * D + ch * 8);
      const float4 b = *reinterpret_cast<const float4*>(sg + (size_t)r * D + ch * 8 + 4);
      uint4 u = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y),
                           pack_bf16(b.z, b.w));
      *reinterpret_cast<uint4*>(s_s + swz(r, ch, RB)) = u;
    }
    for (int c = tid; c < D; c += 128) z_s[c] = sg[D * D + c];
    if (proj)
      for (int e = tid; e < D * CH; e += 128) {
        const int r = e / CH, ch = e % CH;
        *reinterpret_cast<uint4*>(w_s + swz(r, ch, RB)) =
            *reinterpret_cast<const uint4*>(prm.w_p + (size_t)r * D + ch * 8);
      }
  }
  // gate per row: 2 threads per row
  {
    const int r = tid >> 1, half = tid & 1;
    float acc = 0.f;
    if (prm.w_g && r < nvq) {
      const __nv_bfloat16* qr = qg + (size_t)r * D + half * (D / 2);
      const __nv_bfloat16* wg = prm.w_g + (size_t)h * D + half * (D / 2);
      for (int c = 0; c < D / 2; c += 2) {
        float2 a = unpack_bf16(*reinterpret_cast<const uint32_t*>(qr + c));
        float2 b = unpack_bf16(*reinterpret_cast<const uint32_t*>(wg + c));
        acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (half == 0) g_s[r] = prm.w_g ? 1.f / (1.f + __expf(-acc)) : 1.f;
  }
  __syncthreads();
  float proj_acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) proj_acc[n][0] = proj_acc[n][1] = proj_acc[n][2] = proj_acc[n][3] = 0.f;
  const int row0 = 16 * w + (lane >> 2);

  if (use_lin) {
    // denominators phi(q) . Z_i from the same bf16 features
    {
      const int r = tid >> 1, half = tid & 1;
      float acc = 0.f;
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); ++c) {
        const __nv_bfloat16* p =
            reinterpret_cast<const __nv_bfloat16*>(fq_s + swz(r, c >> 3, RB)) + (c & 7);
        acc = fmaf(__bfloat162float(*p), z_s[c], acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      if (half == 0) den_s[r] = acc;
    }
    __syncthreads();
    const uint32_t fq_b = smem_u32(fq_s), s_b = smem_u32(s_s), w_b = smem_u32(w_s),
                   ol_b = smem_u32(ol_s);
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
    const float d0 = den_s[row0], d1 = den_s[row0 + 8];
    const float i0 = d0 > 0.f ? 1.f / d0 : 0.f, i1 = d1 > 0.f ? 1.f / d1 : 0.f;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      num[n][0] *= i0;
      num[n][1] *= i0;
      num[n][2] *= i1;
      num[n][3] *= i1;
    }
    if (proj) {
      // O_l (bf16) -> smem rows of this warp, then O_l W_p
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        const int col = n * 8 + 2 * (lane & 3);
        *reinterpret_cast<uint32_t*>(ol_s + swz(row0, col >> 3, RB) + (col & 7) * 2) =
            pack_bf16(num[n][0], num[n][1]);
        *reinterpret_cast<uint32_t*>(ol_s + swz(row0 + 8, col >> 3, RB) + (col & 7) * 2) =
            pack_bf16(num[n][2], num[n][3]);
      }
      __syncwarp();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(lds_a(ol_b, 16 * w, 2 * ks, RB, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(lds_b_kn(w_b, ks * 16, 2 * n2, RB, lane), b0, b1, b2, b3);
          mma_bf16(proj_acc[2 * n2], a, b0, b1);
          mma_bf16(proj_acc[2 * n2 + 1], a, b2, b3);
        }
      }
    } else {
#pragma unroll
      for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) proj_acc[n][e] = num[n][e];
    }
  }
  // O = O_s + g * proj ; padding rows are zero
  const float g0 = g_s[row0], g1 = g_s[row0 + 8];
  const bool v0 = row0 < nvq, v1 = row0 + 8 < nvq;
  const __nv_bfloat16* osg = prm.os + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
  __nv_bfloat16* og = prm.out + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * (lane & 3);
    float2 s0 = unpack_bf16(*reinterpret_cast<const uint32_t*>(osg + (size_t)row0 * D + col));
    float2 s1 = unpack_bf16(*reinterpret_cast<const uint32_t*>(osg + (size_t)(row0 + 8) * D + col));
    const uint32_t o0 = v0 ? pack_bf16(s0.x + g0 * proj_acc[n][0], s0.y + g0 * proj_acc[n][1]) : 0u;
    const uint32_t o1 = v1 ? pack_bf16(s1.x + g1 * proj_acc[n][2], s1.y + g1 * proj_acc[n][3]) : 0u;
    *reinterpret_cast<uint32_t*>(og + (size_t)row0 * D + col) = o0;
    *reinterpret_cast<uint32_t*>(og + (size_t)(row0 + 8) * D + col) = o1;
  }
}

template <int D>
static cudaError_t launch_epi_t(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  EpiParams prm;
  prm.q = a.q;
  prm.os = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_os);
  prm.ss = reinterpret_cast<const float*>(a.ws + p.off_ss);
  prm.w_p = c.has_proj ? a.w_p : nullptr;
  prm.w_g = c.has_gate ? a.w_g : nullptr;
  prm.out = a.out;
  prm.H = c.H;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = p.nqb;
  prm.dd = p.dd;
  prm.has_marginal = (p.nkb - c.k_h - c.k_l) > 0;
  const int smem = 2 * kBlock * D * 2 + 2 * D * D * 2 + (D + 2 * kBlock) * 4;
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
