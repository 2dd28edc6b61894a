// Per-key-block linear states on the 5th-generation tensor cores.
//
// SLA analysis page (arXiv 2509.24006), comparison table and core-innovation
// paragraph: marginal blocks go through linear attention at O(N d^2). With
// phi = elu + 1 the branch factorises per key block j into the d x d state
// h_j = phi(K_j)^T V_j and the normaliser z_j = sum_t phi(k_t). With a
// projection, W_p is folded in: O_l W_p = phi(q) sum_j phi(K_j)^T (V_j W_p) / den,
// so the kernel stores h'_j = phi(K_j)^T T_j with T_j = V_j W_p.
//
// One CTA per pair of key blocks (128 tokens) of one KV head:
//   1. TMA: K and V (128 tokens x d) and W_p into 128-byte-swizzled tiles.
//   2. T = V W_p on tcgen05 (M = 128 tokens, N = d, K = d) into TMEM.
//   3. Eight worker warps (two per TMEM lane quarter; thread = token row, the
//      two warps of a quarter split the columns): phi(K) in place (padding
//      tokens zero), T back to shared memory as bf16 in the N-major layout V
//      had, z_j by column sums (one block per warp half).
//   4. h'_j = phi(K_j)^T T_j for both blocks (M = d, N = d, K = 64 tokens),
//      phi(K) read M-major straight from the K tile, into TMEM.
//   5. Workers stage h'_j (thread = feature row) as bf16 in the freed K and V
//      tiles, 128-byte swizzled, and one thread writes them with TMA stores.
// Layout: Hs[bkv][j][0 : d*d] = h'_j row-major, [d*d : d*d+d] = z_j, zero up to
// dd (a multiple of 128); rows j in [nkb, nkb_pad) zero.
// For d = 64 the state product still uses M = 128: the second feature panel
// of K is read beyond the tensor and filled with zeros.
// Smooth-K (the SLA critique page's note on the open-source code: zero-mean K):
// phi is applied to k_t - m, m = mean of the head's valid key tokens, computed
// first from the float64 block means of the pooling pass.
#include "common.cuh"
#include "tc.cuh"

namespace sla {

constexpr int kStThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 workers

template <int D>
struct StLayout {
  static constexpr int NP = D / 64;                    // 64-column panels of V, T, W_p
  static constexpr int kKBytes = 2 * 128 * 128;        // K: two feature panels x 128 tokens
  static constexpr int kVBytes = NP * 128 * 128;       // V, then T
  static constexpr int kWBytes = NP * D * 128;         // W_p: N-major panels of D rows
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffW = kOffV + kVBytes;
  static constexpr int kOffBar = kOffW + kWBytes;
  static constexpr int kSmem = kOffBar + 128;
};

struct StateParams {
  __nv_bfloat16* hs;
  int* status;
  int nkb, nkb_pad, dd, n_valid, has_proj;
  int wp_heads;  // 1: one W_p for all heads; H: W_p[h] for KV head h (H_kv == H)
  const float* kmean;  // smooth-K: [B*H_kv][D] mean valid key, or null
};

// m = sum_j n_j kbar_j / N_valid over the blocks of one KV head (n_j valid tokens
// of block j), in float64. 1024 threads: column c = tid % d, part = tid / d sums
// the blocks j = part, part + parts, ...; the parts are added in shared memory
// in a fixed order.
constexpr int kKmeanThreads = 1024;

__global__ void __launch_bounds__(kKmeanThreads)
    kmean_kernel(const double* __restrict__ kbar, float* __restrict__ kmean, int nb, int d, int n_valid) {
  __shared__ double part_sum[kKmeanThreads];
  const int bkv = blockIdx.x, c = threadIdx.x % d, part = threadIdx.x / d, parts = kKmeanThreads / d;
  const double* kb = kbar + (size_t)bkv * nb * d + c;
  double s = 0.0;
#pragma unroll 4
  for (int j = part; j < nb; j += parts) {
    const int nv = n_valid - j * kBlock < kBlock ? n_valid - j * kBlock : kBlock;
    s += (double)nv * kb[(size_t)j * d];
  }
  part_sum[threadIdx.x] = s;
  __syncthreads();
  if (part == 0) {
    double t = 0.0;
    for (int q = 0; q < parts; ++q) t += part_sum[q * d + c];
    kmean[(size_t)bkv * d + c] = (float)(t / (double)n_valid);
  }
}

template <int D>
__global__ void __launch_bounds__(kStThreads, 2)
    state_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmH,
                    StateParams prm) {
  using L = StLayout<D>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  const int j0 = 2 * blockIdx.x, bkv = blockIdx.y;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffBar + 64);  // tmem, abort
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  constexpr int LOADED = 0, T_DONE_MMA = 1, PHI_READY = 2, T_READY = 3, H_DONE = 4;
  constexpr int kWorkerWarps = 8;
  const bool proj = prm.has_proj != 0;
  if (tid == 0) {
    misc[1] = 0;
    tc::mbar_init(bar(LOADED), 1);
    tc::mbar_init(bar(T_DONE_MMA), 1);
    tc::mbar_init(bar(PHI_READY), kWorkerWarps);
    tc::mbar_init(bar(T_READY), kWorkerWarps);
    tc::mbar_init(bar(H_DONE), 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + L::kOffBar + 64, 256);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 1;
  const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sW = sbase + L::kOffW;

  if (warp == 0) {
    if (lane == 0) {
      tc::mbar_expect_tx(bar(LOADED), L::kKBytes + L::kVBytes + (proj ? L::kWBytes : 0));
      for (int p = 0; p < 2; ++p) tc::tma_load_3d(sK + p * 16384, &tmK, bar(LOADED), 64 * p, j0 * kBlock, bkv);
      for (int p = 0; p < L::NP; ++p)
        tc::tma_load_3d(sV + p * 16384, &tmV, bar(LOADED), 64 * p, j0 * kBlock, bkv);
      if (proj)
        for (int p = 0; p < L::NP; ++p)
          tc::tma_load_3d(sW + p * D * 128, &tmW, bar(LOADED), 64 * p, 0, bkv % prm.wp_heads);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = tc::mbar_wait(bar(LOADED), 0, abort);
      tc::fence_after_sync();
      if (ok && proj) {
        // T = V W_p: A = V (K-major over features), B = W_p (N-major)
        constexpr uint32_t kId1 = tc::idesc_bf16(128, D, false, true);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t da = tc::sw128_desc(sV + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
          const uint64_t db = tc::sw128_desc(sW + k * 2048, D * 128, 1024);
          tc::mma_bf16_ss(tmem, da, db, kId1, k > 0);
        }
        tc::mma_commit(bar(T_DONE_MMA));
      }
      if (ok) ok = tc::mbar_wait(bar(PHI_READY), 0, abort);
      if (ok && proj) ok = tc::mbar_wait(bar(T_READY), 0, abort);
      tc::fence_after_sync();
      if (ok) {
        // h'_j = phi(K_j)^T T_j: A = phi(K) M-major (features contiguous), B = T N-major
        constexpr uint32_t kId2 = tc::idesc_bf16(128, D, true, true);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t row_off = (uint32_t)(64 * jj + 16 * kk) * 128;
            const uint64_t da = tc::sw128_desc(sK + row_off, 16384, 1024);
            const uint64_t db = tc::sw128_desc(sV + row_off, 16384, 1024);
            tc::mma_bf16_ss(tmem + jj * D, da, db, kId2, kk > 0);
          }
        tc::mma_commit(bar(H_DONE));
      } else {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    }
  } else {
    // ---- workers: warps 2-9; thread r = token row r of the pair / feature row r;
    // hh = which half of the columns (phi, T) or which block (z, h') this warp takes
    const int quarter = warp & 3;
    const int hh = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(LOADED), 0, abort));
    const int tok = j0 * kBlock + r;
    const bool valid_tok = tok < prm.n_valid;
    if (ok && hh < L::NP) {
      // phi(K) in place on this token's row, feature panel hh: all 8 chunks are
      // loaded before any is written back
      uint4 u[8];
      uint4* row = reinterpret_cast<uint4*>(smem + L::kOffK + hh * 16384 + r * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) u[c] = row[c ^ (r & 7)];
      const float* km = prm.kmean ? prm.kmean + (size_t)bkv * D + 64 * hh : nullptr;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t* w = reinterpret_cast<uint32_t*>(&u[c]);
        float4 m0 = make_float4(0.f, 0.f, 0.f, 0.f), m1 = m0;
        if (km) {
          m0 = *reinterpret_cast<const float4*>(km + 8 * c);
          m1 = *reinterpret_cast<const float4*>(km + 8 * c + 4);
        }
        auto shifted_phi = [&](uint32_t word, float ma, float mb) -> uint32_t {
          const float2 f = unpack_bf16(word);
          return valid_tok ? pack_bf16(phi(f.x - ma), phi(f.y - mb)) : 0u;
        };
        w[0] = shifted_phi(w[0], m0.x, m0.y);
        w[1] = shifted_phi(w[1], m0.z, m0.w);
        w[2] = shifted_phi(w[2], m1.x, m1.y);
        w[3] = shifted_phi(w[3], m1.z, m1.w);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) row[c ^ (r & 7)] = u[c];
      tc::fence_async_smem();
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar(PHI_READY));
    if (ok && proj) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(T_DONE_MMA), 0, abort));
      tc::fence_after_sync();
      if (ok && hh < L::NP) {
        // T row r, columns 64*hh .. +63 (fp32, TMEM) -> bf16 into the V tile (N-major)
        uint32_t v[2][32];
        tc::tmem_ld32(tmem + lane_off + 64 * hh, v[0]);
        tc::tmem_ld32(tmem + lane_off + 64 * hh + 32, v[1]);
        tc::tmem_ld_wait();
        uint4* row = reinterpret_cast<uint4*>(smem + L::kOffV + hh * 16384 + r * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t* vv = v[q >> 2] + 8 * (q & 3);
          row[q ^ (r & 7)] = make_uint4(pack_bf16(__uint_as_float(vv[0]), __uint_as_float(vv[1])),
                                        pack_bf16(__uint_as_float(vv[2]), __uint_as_float(vv[3])),
                                        pack_bf16(__uint_as_float(vv[4]), __uint_as_float(vv[5])),
                                        pack_bf16(__uint_as_float(vv[6]), __uint_as_float(vv[7])));
        }
        tc::fence_async_smem();
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(T_READY));
    }
    // z_j for block hh: column sums of phi(K) over its 64 tokens (all rows written above)
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const int j = j0 + hh;
    if (ok && r < D && j < prm.nkb) {
      const int p = r >> 6, ch = (r & 63) >> 3, e = r & 7;
      const __nv_bfloat16* col = reinterpret_cast<const __nv_bfloat16*>(smem + L::kOffK + p * 16384) + e;
      float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < 64; ++t) {
        const int tt = 64 * hh + t;
        z[t & 7] += __bfloat162float(col[(tt * 128 + ((ch ^ (tt & 7)) << 4)) / 2]);
      }
      const float zs = ((z[0] + z[1]) + (z[2] + z[3])) + ((z[4] + z[5]) + (z[6] + z[7]));
      prm.hs[((size_t)bkv * prm.nkb_pad + j) * prm.dd + D * D + r] = __float2bfloat16(zs);
    }
    __nv_bfloat16* hrow = prm.hs + ((size_t)bkv * prm.nkb_pad + j) * prm.dd;
    if (j >= prm.nkb) {
      // rows past the last key block are zero
      for (int e = r; e < prm.dd / 8; e += 128) reinterpret_cast<uint4*>(hrow)[e] = make_uint4(0, 0, 0, 0);
    } else {
      for (int e = D * D + D + r; e < prm.dd; e += 128) hrow[e] = __float2bfloat16(0.f);
    }
    // every worker has read K (z) before h' overwrites the K and V tiles
    asm volatile("bar.sync 1, 256;" ::: "memory");
    ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(H_DONE), 0, abort));
    tc::fence_after_sync();
    if (ok) {
      // h'_hh row r (feature c1) -> bf16 staged in the K (block 0) or V (block 1)
      // tile: two 64-column panels of 128 rows, 128-byte swizzled
      unsigned char* stage = smem + (hh == 0 ? L::kOffK : L::kOffV);
#pragma unroll
      for (int c64 = 0; c64 < D / 64; ++c64) {
        uint32_t v[2][32];
        tc::tmem_ld32(tmem + lane_off + hh * D + 64 * c64, v[0]);
        tc::tmem_ld32(tmem + lane_off + hh * D + 64 * c64 + 32, v[1]);
        tc::tmem_ld_wait();
        uint4* row = reinterpret_cast<uint4*>(stage + c64 * 16384 + r * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t* vv = v[q >> 2] + 8 * (q & 3);
          row[q ^ (r & 7)] = make_uint4(pack_bf16(__uint_as_float(vv[0]), __uint_as_float(vv[1])),
                                        pack_bf16(__uint_as_float(vv[2]), __uint_as_float(vv[3])),
                                        pack_bf16(__uint_as_float(vv[4]), __uint_as_float(vv[5])),
                                        pack_bf16(__uint_as_float(vv[6]), __uint_as_float(vv[7])));
        }
      }
      tc::fence_async_smem();
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok && quarter == 0 && lane == 0 && j < prm.nkb) {
      // one thread per block: TMA stores of its D x D state (rows c1 < D)
      const uint32_t src = sbase + (hh == 0 ? L::kOffK : L::kOffV);
      for (int c64 = 0; c64 < D / 64; ++c64)
        tc::tma_store_3d(&tmH, src + c64 * 16384, 64 * c64, 0, bkv * prm.nkb_pad + j);
      tc::bulk_commit();
      tc::bulk_wait_all();
    }
    if (!ok) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

template <int D>
static cudaError_t launch_state_t(const Plan& p, const Args& a, cudaStream_t s) {
  using L = StLayout<D>;
  const sla_config& c = p.c;
  CUtensorMap mk, mv, mw;
  const uint64_t rowb = (uint64_t)D * 2, headb = (uint64_t)c.N * D * 2;
  if (!make_tmap_3d(&mk, a.k, D, (uint64_t)c.N_valid, (uint64_t)c.B * c.H_kv, rowb, headb, 64, 128) ||
      !make_tmap_3d(&mv, a.v, D, (uint64_t)c.N_valid, (uint64_t)c.B * c.H_kv, rowb, headb, 64, 128))
    return cudaErrorInvalidValue;
  const bool proj = c.has_proj && a.w_p;
  // h'_j as a [D rows][D columns] tile inside row j of the state array; rows c1 < D only
  CUtensorMap mh;
  if (!make_tmap_3d(&mh, a.ws + p.off_hs, D, D, (uint64_t)c.B * c.H_kv * p.nkb_pad, rowb, (uint64_t)p.dd * 2,
                    64, D))
    return cudaErrorInvalidValue;
  // without a projection the W_p map is never used; encode it over K to keep it valid
  const int wp_heads = proj && c.proj_per_head ? c.H : 1;
  if (!make_tmap_3d(&mw, proj ? (const void*)a.w_p : (const void*)a.k, D, D, (uint64_t)wp_heads, rowb,
                    (uint64_t)D * rowb, 64, D))
    return cudaErrorInvalidValue;
  StateParams prm;
  prm.hs = reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_hs);
  prm.status = a.status;
  prm.nkb = p.nkb;
  prm.nkb_pad = p.nkb_pad;
  prm.dd = p.dd;
  prm.n_valid = c.N_valid;
  prm.has_proj = proj ? 1 : 0;
  prm.wp_heads = wp_heads;
  prm.kmean = nullptr;
  if (c.smooth_k) {
    float* km = reinterpret_cast<float*>(a.ws + p.off_kmean);
    kmean_kernel<<<c.B * c.H_kv, kKmeanThreads, 0, s>>>(reinterpret_cast<const double*>(a.ws + p.off_kbar), km,
                                                          p.nkb, D, c.N_valid);
    prm.kmean = km;
  }
  cudaError_t e = cudaFuncSetAttribute(state_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nkb_pad / 2, c.B * c.H_kv);
  state_tc_kernel<D><<<grid, kStThreads, L::kSmem, s>>>(mk, mv, mw, mh, prm);
  return cudaGetLastError();
}

cudaError_t launch_state(const Plan& p, const Args& a, cudaStream_t s) {
  return p.c.d == 128 ? launch_state_t<128>(p, a, s) : launch_state_t<64>(p, a, s);
}

}  // namespace sla
