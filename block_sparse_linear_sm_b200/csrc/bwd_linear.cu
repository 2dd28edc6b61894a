// Backward pass of the linear branch, the gate and the combine step.
//
// The forward layer (SLA analysis page, arXiv 2509.24006: O = O^s + Proj(O^l),
// linear attention over the marginal blocks; SALAD summary: gated branches)
// writes, per query token t of query block i,
//   u_t = phi(q_t) S'_i / den_t,  den_t = phi(q_t) . Z_i,  S'_i = S_i W_p,
//   O_t = O_s,t + g_t u_t,        g_t = sigmoid(q_t . w_g[h]).
// For L = sum(O * dO), with the routing held fixed:
//   du_t = g_t dO_t, dg_t = dO_t . u_t, dlogit_t = dg_t g_t (1 - g_t)
//   dphi(q_t) = (du_t S'_i^T - (du_t . u_t) Z_i) / den_t
//   dS'_i = sum_t phi(q_t)^T du_t / den_t,  dZ_i = -sum_t phi(q_t) (du_t . u_t) / den_t
//   dq_t (linear and gate part) = dphi(q_t) * phi'(q_t) + dlogit_t w_g[h]
//   dw_g[h] = sum_t dlogit_t q_t
// and the sparse branch needs D_t = dO_t . O_s,t = dO_t . (O_t - g_t u_t).
//
// lin_bwd_kernel: one CTA per pair of query blocks (128 tokens) of one head,
// four warps, thread = token row (TMEM lane). Three tcgen05 phases:
//   1. A_h = phi(Q) S'_h for both blocks (M = 128, N = d, K = d) -> u = A / den
//   2. G_h = DU S'_h^T (DU = du / den, bf16 in shared memory) -> dphi(q)
//   3. dS'_h = phi(Q_h)^T DU_h (M = d features, N = d, K = 64 tokens)
// dS'_i and dZ_i are written as one bf16 row [dS'_i | dZ_i | 0] per (KV head,
// query head of its group, query block), the right-hand side of the transposed
// aggregation dh'_j = sum_i M[i, j] dS'_i.
#include "common.cuh"
#include "tc.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// D_t = dO_t . O_t for layers without a linear branch (O_s = O): one warp per row
// ---------------------------------------------------------------------------
__global__ void delta_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                             float* __restrict__ delta, int64_t rows, int N, int n_valid, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t row = w0; row < rows; row += nw) {
    const int t = (int)(row % N);
    float s = 0.f;
    if (t < n_valid) {
      const uint32_t* o = reinterpret_cast<const uint32_t*>(out + row * d);
      const uint32_t* g = reinterpret_cast<const uint32_t*>(dout + row * d);
      for (int e = lane; e < d / 2; e += 32) {
        const float2 a = unpack_bf16(o[e]), b = unpack_bf16(g[e]);
        s = fmaf(a.x, b.x, fmaf(a.y, b.y, s));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) delta[row] = s;
  }
}

cudaError_t launch_delta(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const int64_t rows = (int64_t)c.B * c.H * c.N;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  delta_kernel<<<(unsigned)blocks, 256, 0, s>>>(a.out, a.dout, reinterpret_cast<float*>(a.bws + bp.off_delta),
                                                 rows, c.N, c.N_valid, c.d);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// linear branch, gate and D_t
// ---------------------------------------------------------------------------
template <int D>
struct LinBwdLayout {
  static constexpr int NP = D / 64;
  static constexpr int kOffF = 0;                         // phi(Q): two feature panels (the second zero for D = 64)
  static constexpr int kOffQ = kOffF + 2 * 16384;         // q
  static constexpr int kOffU = kOffQ + NP * 16384;        // dO, overwritten in place by du / den (bf16)
  static constexpr int kOffO = kOffU + NP * 16384;        // O
  static constexpr int kOffS = kOffO + NP * 16384;        // S'_i of both blocks
  static constexpr int kSBytes = NP * D * 128;            // one S' (D rows x D columns)
  static constexpr int kOffZ = kOffS + 2 * kSBytes;       // Z_i of both blocks (fp32)
  static constexpr int kOffC = kOffZ + 2 * D * 4;         // (du . u) / den per row
  static constexpr int kOffDL = kOffC + 128 * 4;          // dlogit per row
  static constexpr int kOffBar = kOffDL + 128 * 4;
  static constexpr int kSmem = kOffBar + 128;
  static constexpr int kTmemCols = 4 * D;                 // A / dS' (2 D), G (2 D)
};

struct LinBwdParams {
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  const __nv_bfloat16* w_g;  // [H][D] or null
  const float* zs;           // [B*H][nqb][D]
  const float* gate;         // [B*H][N] or null
  float* delta;              // [B*H][N]
  float* dq_acc;             // [B*H][N][D]
  float* dw_g;               // [H][D] or null
  __nv_bfloat16* drow;       // [B*H_kv][group*nqb_pad][dd]
  int* status;
  int H, group, N, n_valid, nqb, nqb_pad, dd, npairs;
};

// byte address of the 16-byte chunk holding columns 8*cidx .. 8*cidx+7 of row r
// in a 128-row tile of 64-column panels with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw_chunk(int panel, int r, int cidx) {
  return (uint32_t)(panel * 16384 + r * 128 + ((cidx ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    lin_bwd_kernel(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmO,
                   const __grid_constant__ CUtensorMap tmG, LinBwdParams prm) {
  using L = LinBwdLayout<D>;
  constexpr int NP = L::NP;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  const int u = blockIdx.x, bh = u / prm.npairs, pr = u % prm.npairs;
  const int b = bh / prm.H, h = bh % prm.H, Hkv = prm.H / prm.group;
  const int bkv = b * Hkv + h / prm.group, gi = h % prm.group;
  const int i_h[2] = {2 * pr, 2 * pr + 1};
  const bool valid_h[2] = {i_h[0] < prm.nqb, i_h[1] < prm.nqb};
  const int nh = valid_h[1] ? 2 : 1;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffBar + 64);  // tmem, abort
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  constexpr int LOADED = 0, MMA1 = 1, MMA2 = 2, MMA3 = 3;
  const uint32_t sF = sbase + L::kOffF, sQ = sbase + L::kOffQ, sU = sbase + L::kOffU, sS = sbase + L::kOffS;
  const float* sZ = reinterpret_cast<const float*>(smem + L::kOffZ);
  float* sC = reinterpret_cast<float*>(smem + L::kOffC);
  float* sDL = reinterpret_cast<float*>(smem + L::kOffDL);
  __nv_bfloat16* row_base = prm.drow + ((size_t)bkv * prm.group + gi) * prm.nqb_pad * prm.dd;

  if (!valid_h[0]) {
    // padding query blocks of the aggregation's right-hand side: zero rows
    for (int hf = 0; hf < 2; ++hf) {
      if (i_h[hf] >= prm.nqb_pad) continue;
      uint4* dst = reinterpret_cast<uint4*>(row_base + (size_t)i_h[hf] * prm.dd);
      for (int e = tid; e < prm.dd / 8; e += 128) dst[e] = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  if (tid == 0) {
    misc[1] = 0;
    for (int k = 0; k < 4; ++k) tc::mbar_init(bar(k), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(sbase + L::kOffBar + 64, L::kTmemCols);
    tc::tmem_relinquish();
  }
  if (D == 64) {
    // features 64..127 of the M-major phi(Q) operand (M = 128) read as zero
    uint4* z = reinterpret_cast<uint4*>(smem + L::kOffF + 16384);
    for (int e = tid; e < 16384 / 16; e += 128) z[e] = make_uint4(0, 0, 0, 0);
    tc::fence_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 1;

  if (tid == 0) {
    tc::mbar_expect_tx(bar(LOADED), 8 * NP * 8192 + nh * (L::kSBytes + D * 4));
    for (int hf = 0; hf < 2; ++hf)
      for (int p = 0; p < NP; ++p) {
        const uint32_t o = p * 16384 + hf * 8192;
        tc::tma_load_3d(sF + o, &tmF, bar(LOADED), 64 * p, i_h[hf] * kBlock, bh);
        tc::tma_load_3d(sQ + o, &tmQ, bar(LOADED), 64 * p, i_h[hf] * kBlock, bh);
        tc::tma_load_3d(sU + o, &tmG, bar(LOADED), 64 * p, i_h[hf] * kBlock, bh);
        tc::tma_load_3d(sbase + L::kOffO + o, &tmO, bar(LOADED), 64 * p, i_h[hf] * kBlock, bh);
      }
    for (int hf = 0; hf < nh; ++hf) {
      for (int p = 0; p < NP; ++p)
        tc::tma_load_3d(sS + hf * L::kSBytes + p * D * 128, &tmS, bar(LOADED), 64 * p, 0, bh * prm.nqb + i_h[hf]);
      tc::bulk_load(sbase + L::kOffZ + hf * D * 4, prm.zs + ((size_t)bh * prm.nqb + i_h[hf]) * D, D * 4,
                    bar(LOADED));
    }
  }
  bool ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(LOADED), 0, abort));
  tc::fence_after_sync();
  // phase 1: A_h = phi(Q) S'_h (B = S' N-major)
  if (warp == 0) {
    if (ok && tc::elect_one()) {
      constexpr uint32_t kId = tc::idesc_bf16(128, D, false, true);
      const uint64_t dF = tc::sw128_desc(sF, 16, 1024);
      for (int hf = 0; hf < nh; ++hf) {
        const uint64_t dS = tc::sw128_desc(sS + hf * L::kSBytes, D * 128, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tmem + hf * D, dF + (uint32_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                          dS + (uint32_t)((k * 2048) >> 4), kId, k > 0);
      }
      tc::mma_commit(bar(MMA1));
    }
    __syncwarp();
  }

  const int r = tid, hf = r >> 6;
  const int t = i_h[hf] * kBlock + (r & 63);
  const bool vrow = valid_h[hf] && t < prm.n_valid;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const float* zrow = sZ + hf * D;
  // den = phi(q) . Z_i from the shared tiles
  float den = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(smem + L::kOffF + sw_chunk(p, r, c));
      const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16(ws4[e]);
        den = fmaf(f.x, zrow[64 * p + 8 * c + 2 * e], fmaf(f.y, zrow[64 * p + 8 * c + 2 * e + 1], den));
      }
    }
  const float inv_den = (vrow && den > 0.f) ? 1.f / den : 0.f;
  const float gt = (prm.gate != nullptr && vrow) ? prm.gate[(size_t)bh * prm.N + t] : 1.f;
  ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA1), 0, abort));
  tc::fence_after_sync();
  float dg = 0.f, dt = 0.f, cu = 0.f;
  if (ok) {
    // O and dO rows from the tiles the loads brought in (rows past N_valid read as zero)
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t av[32];
      tc::tmem_ld32(tmem + lane_off + hf * D + 32 * ch, av);
      tc::tmem_ld_wait();
      uint32_t ow[16], gw[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint32_t off = sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4);
        const uint4 o4 = vrow ? *reinterpret_cast<const uint4*>(smem + L::kOffO + off) : make_uint4(0, 0, 0, 0);
        const uint4 g4 = vrow ? *reinterpret_cast<const uint4*>(smem + L::kOffU + off) : make_uint4(0, 0, 0, 0);
        ow[4 * q4] = o4.x; ow[4 * q4 + 1] = o4.y; ow[4 * q4 + 2] = o4.z; ow[4 * q4 + 3] = o4.w;
        gw[4 * q4] = g4.x; gw[4 * q4 + 1] = g4.y; gw[4 * q4 + 2] = g4.z; gw[4 * q4 + 3] = g4.w;
      }
      uint32_t du[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 o = unpack_bf16(ow[e]), g = unpack_bf16(gw[e]);
        // rows without a state (padding, no marginal block) never read TMEM values
        const float u0 = inv_den != 0.f ? __uint_as_float(av[2 * e]) * inv_den : 0.f;
        const float u1 = inv_den != 0.f ? __uint_as_float(av[2 * e + 1]) * inv_den : 0.f;
        dg = fmaf(g.x, u0, fmaf(g.y, u1, dg));
        dt = fmaf(g.x, o.x - gt * u0, fmaf(g.y, o.y - gt * u1, dt));
        const float d0 = gt * g.x, d1 = gt * g.y;
        cu = fmaf(d0, u0, fmaf(d1, u1, cu));
        du[e] = pack_bf16(d0 * inv_den, d1 * inv_den);
      }
      // columns 32ch .. 32ch+31: panel (32ch)/64, chunks ((32ch) % 64)/8 .. +3
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4*>(smem + L::kOffU + sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4)) =
            make_uint4(du[4 * q4], du[4 * q4 + 1], du[4 * q4 + 2], du[4 * q4 + 3]);
    }
  }
  if (valid_h[hf]) prm.delta[(size_t)bh * prm.N + t] = vrow ? dt : 0.f;
  const float cp = cu * inv_den;  // (du . u) / den
  const float dlogit = (prm.gate != nullptr && vrow) ? dg * gt * (1.f - gt) : 0.f;
  sC[r] = cp;
  sDL[r] = dlogit;
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // phase 2: G_h = DU S'_h^T (B = S' K-major); phase 3: dS'_h = phi(Q_h)^T DU_h into the A columns
  if (warp == 0) {
    if (ok && tc::elect_one()) {
      constexpr uint32_t kId2 = tc::idesc_bf16(128, D, false, false);
      constexpr uint32_t kId3 = tc::idesc_bf16(128, D, true, true);
      const uint64_t dU = tc::sw128_desc(sU, 16, 1024);
      for (int x = 0; x < nh; ++x) {
        const uint64_t dS = tc::sw128_desc(sS + x * L::kSBytes, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tmem + 2 * D + x * D, dU + (uint32_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                          dS + (uint32_t)(((k >> 2) * (D * 128) + (k & 3) * 32) >> 4), kId2, k > 0);
      }
      tc::mma_commit(bar(MMA2));
      for (int x = 0; x < nh; ++x) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t off = (uint32_t)(64 * x + 16 * kk) * 128;
          tc::mma_bf16_ss(tmem + x * D, tc::sw128_desc(sF + off, 16384, 1024),
                          tc::sw128_desc(sU + off, 16384, 1024), kId3, kk > 0);
        }
      }
      tc::mma_commit(bar(MMA3));
    }
    __syncwarp();
  }
  ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA2), 0, abort));
  tc::fence_after_sync();
  if (ok && valid_h[hf]) {
    // dq_t = (G - cp Z) * phi'(q) + dlogit w_g[h]
    float4* dst = reinterpret_cast<float4*>(prm.dq_acc + ((size_t)bh * prm.N + t) * D);
    const __nv_bfloat16* wg = prm.w_g ? prm.w_g + (size_t)h * D : nullptr;
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t gv[32];
      tc::tmem_ld32(tmem + lane_off + 2 * D + hf * D + 32 * ch, gv);
      tc::tmem_ld_wait();
      float res[32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint4 w = *reinterpret_cast<const uint4*>(smem + L::kOffQ +
                                                        sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4));
        const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 qv = unpack_bf16(ws4[e]);
          const int j = 8 * q4 + 2 * e, col = 32 * ch + j;
          const float dphi0 = __uint_as_float(gv[j]) - cp * zrow[col];
          const float dphi1 = __uint_as_float(gv[j + 1]) - cp * zrow[col + 1];
          float r0 = dphi0 * (qv.x > 0.f ? 1.f : __expf(qv.x));
          float r1 = dphi1 * (qv.y > 0.f ? 1.f : __expf(qv.y));
          if (wg) {
            r0 = fmaf(dlogit, __bfloat162float(wg[col]), r0);
            r1 = fmaf(dlogit, __bfloat162float(wg[col + 1]), r1);
          }
          res[j] = vrow ? r0 : 0.f;
          res[j + 1] = vrow ? r1 : 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[8 * ch + j] = make_float4(res[4 * j], res[4 * j + 1], res[4 * j + 2], res[4 * j + 3]);
    }
  }
  ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA3), 0, abort));
  tc::fence_after_sync();
  // thread r = feature row c of dS'_h; dZ_h[c] = -sum over the block's rows of phi(q)[c] cp
  for (int x = 0; x < 2; ++x) {
    if (i_h[x] >= prm.nqb_pad) continue;
    __nv_bfloat16* dst = row_base + (size_t)i_h[x] * prm.dd;
    if (!valid_h[x] || !ok) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
      for (int e = tid; e < prm.dd / 8; e += 128) d4[e] = make_uint4(0, 0, 0, 0);
      continue;
    }
    if (r < D) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)r * D);
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t sv[32];
        tc::tmem_ld32(tmem + lane_off + x * D + 32 * ch, sv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          d4[4 * ch + q4] = make_uint4(pack_bf16(__uint_as_float(sv[8 * q4]), __uint_as_float(sv[8 * q4 + 1])),
                                       pack_bf16(__uint_as_float(sv[8 * q4 + 2]), __uint_as_float(sv[8 * q4 + 3])),
                                       pack_bf16(__uint_as_float(sv[8 * q4 + 4]), __uint_as_float(sv[8 * q4 + 5])),
                                       pack_bf16(__uint_as_float(sv[8 * q4 + 6]), __uint_as_float(sv[8 * q4 + 7])));
      }
      float z = 0.f;
      const int p = r >> 6, cidx = (r & 63) >> 3, e = r & 7;
      for (int rr = 64 * x; rr < 64 * x + 64; ++rr) {
        const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(smem + L::kOffF + sw_chunk(p, rr, cidx));
        z = fmaf(__bfloat162float(row[e]), sC[rr], z);
      }
      dst[D * D + r] = __float2bfloat16(-z);
    }
    for (int e = D * D + D + tid; e < prm.dd; e += 128) dst[e] = __float2bfloat16(0.f);
  }
  if (prm.dw_g != nullptr && ok && r < D) {
    // dw_g[h][c] += sum over the unit's rows of dlogit q[c]
    float s = 0.f;
    const int p = r >> 6, cidx = (r & 63) >> 3, e = r & 7;
    for (int rr = 0; rr < 128; ++rr) {
      const __nv_bfloat16* row = reinterpret_cast<const __nv_bfloat16*>(smem + L::kOffQ + sw_chunk(p, rr, cidx));
      s = fmaf(__bfloat162float(row[e]), sDL[rr], s);
    }
    atomicAdd(prm.dw_g + (size_t)h * D + r, s);
  }
  if (!ok && lane == 0) {
    *abort = 1;
    report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
static cudaError_t launch_lin_bwd_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  using L = LinBwdLayout<D>;
  const sla_config& c = p.c;
  const uint64_t rowb = (uint64_t)D * 2, headb = (uint64_t)c.N * D * 2, bh = (uint64_t)c.B * c.H;
  CUtensorMap mf, mq, ms, mo, mg;
  if (!make_tmap_3d(&mf, a.ws + p.off_phiq, D, (uint64_t)c.N_valid, bh, rowb, headb, 64, 64) ||
      !make_tmap_3d(&mq, a.q, D, (uint64_t)c.N_valid, bh, rowb, headb, 64, 64) ||
      !make_tmap_3d(&mo, a.out, D, (uint64_t)c.N_valid, bh, rowb, headb, 64, 64) ||
      !make_tmap_3d(&mg, a.dout, D, (uint64_t)c.N_valid, bh, rowb, headb, 64, 64) ||
      !make_tmap_3d(&ms, a.ws + p.off_ss, D, D, bh * p.nqb, rowb, (uint64_t)D * D * 2, 64, D))
    return cudaErrorInvalidValue;
  LinBwdParams prm;
  prm.out = a.out;
  prm.dout = a.dout;
  prm.w_g = c.has_gate ? a.w_g : nullptr;
  prm.zs = reinterpret_cast<const float*>(a.ws + p.off_zs);
  prm.gate = c.has_gate ? reinterpret_cast<const float*>(a.ws + p.off_gate) : nullptr;
  prm.delta = reinterpret_cast<float*>(a.bws + bp.off_delta);
  prm.dq_acc = reinterpret_cast<float*>(a.bws + bp.off_dqacc);
  prm.dw_g = c.has_gate ? a.dw_g : nullptr;
  prm.drow = reinterpret_cast<__nv_bfloat16*>(a.bws + bp.off_drow);
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nqb = p.nqb;
  prm.nqb_pad = p.nqb_pad;
  prm.dd = p.dd;
  prm.npairs = p.nqb_pad / 2;  // units past nqb write the zero padding rows
  cudaError_t e = cudaFuncSetAttribute(lin_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  lin_bwd_kernel<D><<<(unsigned)(bh * prm.npairs), 128, L::kSmem, s>>>(mf, mq, ms, mo, mg, prm);
  return cudaGetLastError();
}

cudaError_t launch_lin_bwd(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  return p.c.d == 128 ? launch_lin_bwd_t<128>(p, bp, a, s) : launch_lin_bwd_t<64>(p, bp, a, s);
}

// ---------------------------------------------------------------------------
// transposed aggregation mask: maskT[bkv][j][g * nqb_pad + i] = mmask[head g of bkv][i][j]
// (32 x 32 tiles through shared memory; the padding of mmask is zero)
// ---------------------------------------------------------------------------
__global__ void mask_t_kernel(const uint16_t* __restrict__ mm, uint16_t* __restrict__ mt, int H, int group,
                              int nqb_pad, int nkb_pad) {
  __shared__ uint16_t tile[32][33];
  const int bh = blockIdx.z, b = bh / H, h = bh % H;
  const int bkv = b * (H / group) + h / group, g = h % group;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  const uint16_t* src = mm + (size_t)bh * nqb_pad * nkb_pad;
  for (int y = ty; y < 32; y += 8) tile[y][tx] = src[(size_t)(i0 + y) * nkb_pad + j0 + tx];
  __syncthreads();
  const size_t rows_t = (size_t)group * nqb_pad;
  uint16_t* dst = mt + (size_t)bkv * nkb_pad * rows_t + (size_t)g * nqb_pad + i0;
  for (int y = ty; y < 32; y += 8) dst[(size_t)(j0 + y) * rows_t + tx] = tile[tx][y];
}

cudaError_t launch_mask_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  dim3 grid(p.nkb_pad / 32, p.nqb_pad / 32, c.B * c.H);
  mask_t_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(a.ws + p.off_mmask),
                                     reinterpret_cast<uint16_t*>(a.bws + bp.off_maskt), c.H, p.group, p.nqb_pad,
                                     p.nkb_pad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// per-key-block states, backward
// ---------------------------------------------------------------------------
// The forward stores h'_j = phi(K_j)^T T_j with T_j = V_j W_p and z_j = sum_t phi(k_t).
// Given dh'_j and dz_j (the transposed aggregation of dS'_i, dZ_i):
//   dT_j = phi(K_j) dh'_j          dphi(K_j) = T_j dh'_j^T + 1 dz_j^T
//   dV_j = dT_j W_p^T               dW_p += V_j^T dT_j
//   dk_t = dphi(k_t) * phi'(k_t) (valid tokens; 0 for padding)
// One CTA per pair of key blocks (128 tokens) of one KV head, four warps,
// thread = token row (or feature row for dW_p). tcgen05 phases:
//   0. T = V W_p                                  (M = 128 tokens, N = D, K = D)
//   1. dT_h = phi(K) dh'_h, dphi(K)_h = T dh'_h^T  (per block h of the pair)
//   2. dV = dT W_p^T, dW_p = V^T dT                (dW_p: M = 128 features, K = 128 tokens)
// Without a projection T = V, dV = dT and phase 2 is skipped.
template <int D>
struct StBwdLayout {
  static constexpr int NP = D / 64;
  static constexpr int kOffK = 0;                    // K, then phi(K): two feature panels
  static constexpr int kOffV = kOffK + 2 * 16384;    // V: two feature panels (M-major operand of dW_p)
  static constexpr int kOffT = kOffV + 2 * 16384;    // T, then dT (bf16)
  static constexpr int kOffW = kOffT + NP * 16384;   // W_p, N-major panels of D rows
  static constexpr int kHBytes = NP * D * 128;       // one dh' (D rows x D columns)
  static constexpr int kOffH = kOffW + NP * D * 128;
  static constexpr int kOffZ = kOffH + 2 * kHBytes;  // dz of both blocks (fp32)
  static constexpr int kOffBar = kOffZ + 2 * D * 4;
  static constexpr int kSmem = kOffBar + 128;
  static constexpr int kTmemCols = 4 * D;            // dT / dV, dW_p (2 D); T, then dphi(K) (2 D)
};

struct StBwdParams {
  const __nv_bfloat16* k;  // [B*H_kv][N][D]
  const float* dz;         // [B*H_kv][nkb][D]
  float* dk_acc;           // [B*H_kv][N][D]
  float* dv_acc;
  float* dwp_part;         // [B*H_kv*npairs][D][D]: this CTA's dW_p partial, or null
  const float* kmean;      // smooth-K: [B*H_kv][D] mean valid key (phi and phi' of k - m), or null
  int* status;
  int N, n_valid, nkb, npairs, has_proj, wp_heads;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    state_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmH,
                     StBwdParams prm) {
  using L = StBwdLayout<D>;
  constexpr int NP = L::NP;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  const int bkv = blockIdx.x / prm.npairs, pr = blockIdx.x % prm.npairs;
  const int j_h[2] = {2 * pr, 2 * pr + 1};
  const int nh = j_h[1] < prm.nkb ? 2 : 1;
  const bool proj = prm.has_proj != 0;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffBar + 64);
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  constexpr int LOADED = 0, MMA0 = 1, MMA1 = 2, MMA2 = 3;
  const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sT = sbase + L::kOffT, sW = sbase + L::kOffW,
                 sH = sbase + L::kOffH;
  const float* sZ = reinterpret_cast<const float*>(smem + L::kOffZ);
  if (tid == 0) {
    misc[1] = 0;
    for (int k = 0; k < 4; ++k) tc::mbar_init(bar(k), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(sbase + L::kOffBar + 64, L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 1;
  if (tid == 0) {
    // K and V always as two feature panels: for D = 64 the second reads past the
    // tensor's columns and is zero-filled
    tc::mbar_expect_tx(bar(LOADED), 4 * 16384 + (proj ? NP * D * 128 : 0) + nh * (L::kHBytes + D * 4));
    for (int p = 0; p < 2; ++p) {
      tc::tma_load_3d(sK + p * 16384, &tmK, bar(LOADED), 64 * p, j_h[0] * kBlock, bkv);
      tc::tma_load_3d(sV + p * 16384, &tmV, bar(LOADED), 64 * p, j_h[0] * kBlock, bkv);
    }
    if (proj)
      for (int p = 0; p < NP; ++p) tc::tma_load_3d(sW + p * D * 128, &tmW, bar(LOADED), 64 * p, 0, bkv % prm.wp_heads);
    for (int x = 0; x < nh; ++x) {
      for (int p = 0; p < NP; ++p)
        tc::tma_load_3d(sH + x * L::kHBytes + p * D * 128, &tmH, bar(LOADED), 64 * p, 0, bkv * prm.nkb + j_h[x]);
      tc::bulk_load(sbase + L::kOffZ + x * D * 4, prm.dz + ((size_t)bkv * prm.nkb + j_h[x]) * D, D * 4, bar(LOADED));
    }
  }
  bool ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(LOADED), 0, abort));
  tc::fence_after_sync();
  if (warp == 0) {
    if (ok && proj && tc::elect_one()) {
      // T = V W_p: A = V K-major, B = W_p N-major
      constexpr uint32_t kId = tc::idesc_bf16(128, D, false, true);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_bf16_ss(tmem + 2 * D, tc::sw128_desc(sV + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                        tc::sw128_desc(sW + k * 2048, D * 128, 1024), kId, k > 0);
      tc::mma_commit(bar(MMA0));
    }
    __syncwarp();
  }
  const int r = tid, hf = r >> 6;
  const int tok = j_h[0] * kBlock + r;
  const bool vtok = tok < prm.n_valid;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (ok) {
    // phi(K) (smooth-K: phi(K - m)) in place on this token's row (padding tokens zero)
    const float* km = prm.kmean ? prm.kmean + (size_t)bkv * D : nullptr;
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4* w = reinterpret_cast<uint4*>(smem + L::kOffK + sw_chunk(p, r, c));
        uint4 x = *w;
        uint32_t* xs = reinterpret_cast<uint32_t*>(&x);
        float mv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (km) {
          const float4 m0 = *reinterpret_cast<const float4*>(km + 64 * p + 8 * c);
          const float4 m1 = *reinterpret_cast<const float4*>(km + 64 * p + 8 * c + 4);
          mv[0] = m0.x; mv[1] = m0.y; mv[2] = m0.z; mv[3] = m0.w;
          mv[4] = m1.x; mv[5] = m1.y; mv[6] = m1.z; mv[7] = m1.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16(xs[e]);
          xs[e] = vtok ? pack_bf16(phi(f.x - mv[2 * e]), phi(f.y - mv[2 * e + 1])) : 0u;
        }
        *w = x;
      }
  }
  if (proj) {
    ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA0), 0, abort));
    tc::fence_after_sync();
    if (ok)
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tc::tmem_ld32(tmem + lane_off + 2 * D + 32 * ch, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<uint4*>(smem + L::kOffT + sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4)) =
              make_uint4(pack_bf16(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
      }
  }
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t sTT = proj ? sT : sV;  // T
  if (warp == 0) {
    if (ok && tc::elect_one()) {
      constexpr uint32_t kIdA = tc::idesc_bf16(128, D, false, true);
      constexpr uint32_t kIdB = tc::idesc_bf16(128, D, false, false);
      for (int x = 0; x < nh; ++x) {
        const uint32_t h0 = sH + x * L::kHBytes;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tmem + x * D, tc::sw128_desc(sK + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                          tc::sw128_desc(h0 + k * 2048, D * 128, 1024), kIdA, k > 0);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tmem + 2 * D + x * D, tc::sw128_desc(sTT + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                          tc::sw128_desc(h0 + (k >> 2) * (D * 128) + (k & 3) * 32, 16, 1024), kIdB, k > 0);
      }
      tc::mma_commit(bar(MMA1));
    }
    __syncwarp();
  }
  ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA1), 0, abort));
  tc::fence_after_sync();
  const bool live = hf < nh;  // the block of this row exists
  float* dv_row = prm.dv_acc + ((size_t)bkv * prm.N + (live ? tok : 0)) * D;
  if (ok && live) {
    // dT row: bf16 into the T tile (T is consumed), or dV = dT without a projection
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t v[32];
      tc::tmem_ld32(tmem + lane_off + hf * D + 32 * ch, v);
      tc::tmem_ld_wait();
      if (proj) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<uint4*>(smem + L::kOffT + sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4)) =
              make_uint4(pack_bf16(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                         pack_bf16(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
      } else {
        float4* d4 = reinterpret_cast<float4*>(dv_row + 32 * ch);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = vtok ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  if (proj && !live) {
    // the absent block's rows of dT are zero (they enter dW_p = V^T dT)
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(smem + L::kOffT + sw_chunk(p, r, c)) = make_uint4(0, 0, 0, 0);
  }
  if (proj) {
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) {
      if (ok && tc::elect_one()) {
        // dV = dT W_p^T (B = W_p K-major); dW_p = V^T dT (A = V M-major, B = dT N-major)
        constexpr uint32_t kIdC = tc::idesc_bf16(128, D, false, false);
        constexpr uint32_t kIdD = tc::idesc_bf16(128, D, true, true);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tmem, tc::sw128_desc(sT + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                          tc::sw128_desc(sW + (k >> 2) * (D * 128) + (k & 3) * 32, 16, 1024), kIdC, k > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16_ss(tmem + D, tc::sw128_desc(sV + kk * 16 * 128, 16384, 1024),
                          tc::sw128_desc(sT + kk * 16 * 128, 16384, 1024), kIdD, kk > 0);
        tc::mma_commit(bar(MMA2));
      }
      __syncwarp();
    }
  }
  // dk = (T dh'^T + dz) * phi'(k), phi'(k) = 1 for k > 0 and e^k = phi(k) otherwise, read off the
  // phi(K) tile in shared memory (phi(k) >= 1 exactly when k > 0 up to the bf16 rounding of phi)
  if (ok && live) {
    float* dk_row = prm.dk_acc + ((size_t)bkv * prm.N + tok) * D;
    const float* z = sZ + hf * D;
#pragma unroll 1
    for (int ch = 0; ch < D / 32; ++ch) {
      uint32_t v[32];
      tc::tmem_ld32(tmem + lane_off + 2 * D + hf * D + 32 * ch, v);
      tc::tmem_ld_wait();
      float res[32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint4 kw = *reinterpret_cast<const uint4*>(smem + L::kOffK +
                                                         sw_chunk((32 * ch) >> 6, r, (((32 * ch) & 63) >> 3) + q4));
        const uint32_t ks[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fk = unpack_bf16(ks[e]);
          const int j = 8 * q4 + 2 * e, col = 32 * ch + j;
          res[j] = vtok ? (__uint_as_float(v[j]) + z[col]) * fminf(fk.x, 1.f) : 0.f;
          res[j + 1] = vtok ? (__uint_as_float(v[j + 1]) + z[col + 1]) * fminf(fk.y, 1.f) : 0.f;
        }
      }
      float4* d4 = reinterpret_cast<float4*>(dk_row + 32 * ch);
#pragma unroll
      for (int j = 0; j < 8; ++j) d4[j] = make_float4(res[4 * j], res[4 * j + 1], res[4 * j + 2], res[4 * j + 3]);
    }
  }
  if (proj) {
    ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(MMA2), 0, abort));
    tc::fence_after_sync();
    if (ok && live) {
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tc::tmem_ld32(tmem + lane_off + 32 * ch, v);
        tc::tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(dv_row + 32 * ch);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          d4[j] = vtok ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (r < D) {
      // dW_p row c of this CTA's 128 tokens, as a partial (reduced by dwp_reduce_kernel)
      float4* wrow = reinterpret_cast<float4*>(prm.dwp_part + ((size_t)blockIdx.x * D + r) * D);
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        if (ok) {
          tc::tmem_ld32(tmem + lane_off + D + 32 * ch, v);
          tc::tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          wrow[8 * ch + j] = ok ? make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                              __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  if (!ok && lane == 0) {
    *abort = 1;
    report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Smooth-K: column sums of the linear-branch dk (the gradient with respect to k - m) over
// the valid tokens of each KV head, in two fixed-order passes (deterministic):
// kcol_part_kernel grid (B*H_kv, kKcolSeg): one thread per column sums a segment of rows;
// kcol_reduce_kernel adds the segments in order and scales by -1 / N_valid.
constexpr int kKcolSeg = 64;

__global__ void kcol_part_kernel(const float* __restrict__ dk_acc, float* __restrict__ part, int N, int n_valid,
                                 int d) {
  const int bkv = blockIdx.x, seg = blockIdx.y, c = threadIdx.x;
  if (c >= d) return;
  const int per = (n_valid + kKcolSeg - 1) / kKcolSeg;
  const int t0 = seg * per, t1 = min(n_valid, t0 + per);
  const float* src = dk_acc + (size_t)bkv * N * d + c;
  float acc = 0.f;
  for (int t = t0; t < t1; ++t) acc += src[(size_t)t * d];
  part[((size_t)bkv * kKcolSeg + seg) * d + c] = acc;
}

__global__ void kcol_reduce_kernel(const float* __restrict__ part, float* __restrict__ kcol, int n_valid, int d) {
  const int bkv = blockIdx.x, c = threadIdx.x;
  if (c >= d) return;
  float acc = 0.f;
  for (int seg = 0; seg < kKcolSeg; ++seg) acc += part[((size_t)bkv * kKcolSeg + seg) * d + c];
  kcol[(size_t)bkv * d + c] = -acc / (float)n_valid;
}

// dW_p[w] = sum of the partials of the units whose KV head uses W_p[w] (w = bkv % wp_heads).
// grid (D*D/4 / 128, segments, wp_heads): each thread sums one float4 column over a
// segment of the units and adds it to the gradient.
__global__ void dwp_reduce_kernel(const float4* __restrict__ part, float* __restrict__ dw_p, int units,
                                  int npairs, int wp_heads, int dsq4) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x, w = blockIdx.z;
  if (e >= dsq4) return;
  const int seg = gridDim.y, per = (units + seg - 1) / seg;
  const int u0 = blockIdx.y * per, u1 = min(units, u0 + per);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int u = u0; u < u1; ++u) {
    if ((u / npairs) % wp_heads != w) continue;
    const float4 x = part[(size_t)u * dsq4 + e];
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  }
  float* dst = dw_p + ((size_t)w * dsq4 + e) * 4;
  atomicAdd(dst, acc.x);
  atomicAdd(dst + 1, acc.y);
  atomicAdd(dst + 2, acc.z);
  atomicAdd(dst + 3, acc.w);
}

template <int D>
static cudaError_t launch_state_bwd_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  using L = StBwdLayout<D>;
  const sla_config& c = p.c;
  const uint64_t rowb = (uint64_t)D * 2, headb = (uint64_t)c.N * D * 2, bkv = (uint64_t)c.B * c.H_kv;
  const bool proj = c.has_proj != 0;
  const int wp_heads = proj && c.proj_per_head ? c.H : 1;
  CUtensorMap mk, mv, mw, mh;
  if (!make_tmap_3d(&mk, a.k, D, (uint64_t)c.N_valid, bkv, rowb, headb, 64, 128) ||
      !make_tmap_3d(&mv, a.v, D, (uint64_t)c.N_valid, bkv, rowb, headb, 64, 128) ||
      !make_tmap_3d(&mw, proj ? (const void*)a.w_p : (const void*)a.k, D, D, (uint64_t)wp_heads, rowb,
                    (uint64_t)D * rowb, 64, D) ||
      !make_tmap_3d(&mh, a.bws + bp.off_dh, D, D, bkv * p.nkb, rowb, (uint64_t)D * D * 2, 64, D))
    return cudaErrorInvalidValue;
  StBwdParams prm;
  prm.k = a.k;
  prm.dz = reinterpret_cast<const float*>(a.bws + bp.off_dz);
  prm.dk_acc = reinterpret_cast<float*>(a.bws + bp.off_dkacc);
  prm.dv_acc = reinterpret_cast<float*>(a.bws + bp.off_dvacc);
  prm.dwp_part = proj ? reinterpret_cast<float*>(a.bws + bp.off_dwp) : nullptr;
  prm.status = a.status;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nkb = p.nkb;
  prm.npairs = (p.nkb + 1) / 2;
  prm.has_proj = proj ? 1 : 0;
  prm.wp_heads = wp_heads;
  prm.kmean = c.smooth_k ? reinterpret_cast<const float*>(a.ws + p.off_kmean) : nullptr;
  cudaError_t e = cudaFuncSetAttribute(state_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  const int units = (int)bkv * prm.npairs;
  state_bwd_kernel<D><<<units, 128, L::kSmem, s>>>(mk, mv, mw, mh, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (c.smooth_k) {
    float* part = reinterpret_cast<float*>(a.bws + bp.off_kcolp);
    kcol_part_kernel<<<dim3((unsigned)bkv, kKcolSeg), D, 0, s>>>(prm.dk_acc, part, c.N, c.N_valid, D);
    kcol_reduce_kernel<<<(unsigned)bkv, D, 0, s>>>(part, reinterpret_cast<float*>(a.bws + bp.off_kcol), c.N_valid, D);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!proj) return cudaSuccess;
  dim3 grid((D * D / 4 + 127) / 128, 64, wp_heads);
  dwp_reduce_kernel<<<grid, 128, 0, s>>>(reinterpret_cast<const float4*>(prm.dwp_part), a.dw_p, units,
                                         prm.npairs, wp_heads, D * D / 4);
  return cudaGetLastError();
}

cudaError_t launch_state_bwd(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  return p.c.d == 128 ? launch_state_bwd_t<128>(p, bp, a, s) : launch_state_bwd_t<64>(p, bp, a, s);
}

}  // namespace sla
