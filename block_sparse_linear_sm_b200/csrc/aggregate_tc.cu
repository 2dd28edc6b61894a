// Aggregation of the linear branch on the 5th-generation tensor cores.
//
// For every query head, S_i = sum over the marginal blocks j of row i of the
// per-block state h_j (d x d, with W_p folded in) and Z_i = sum of z_j (SLA
// analysis page, arXiv 2509.24006: linear attention over the marginal blocks).
// Written as one GEMM per head:
//
//   C[i, :] = sum_j M[i, j] * Hs[j, :]     M: 0/1 marginal mask (exact in bf16)
//
// with C = [S_i | Z_i] row by row.
//
// Persistent kernel, one CTA per SM. Output tiles are 128 (query blocks) x 256
// (state columns), K = key blocks in steps of 64. The tile order runs the
// query-block tiles of one column tile next to each other, so a tile of states
// comes from HBM once and from L2 for its other users. TMEM holds two
// accumulators (2 x 256 columns): the MMA warp fills one while the epilogue
// warps drain the other, so a tile's epilogue (TMEM to registers to a
// 128-byte-swizzled staging buffer to TMA stores) overlaps the next tile's
// main loop.
//
// Warps: 0 = TMA producer (A = mask, K-major; B = states, N-major; 3-stage
// ring), 1 = TMEM owner and MMA issuer (whole warp, one elected lane issues),
// 2-5 = epilogue (S_i columns to bf16 through the staging buffer, Z_i columns
// straight to HBM as fp32, padding columns dropped).
#include "common.cuh"
#include "tc.cuh"

namespace sla {

constexpr int kAgStages = 3;
constexpr int kAgThreads = 192;
constexpr int kAgBM = 128, kAgBN = 256;
constexpr int kAgA = kAgBM * 64 * 2;          // mask tile: 128 rows x 64 k
constexpr int kAgB = 64 * kAgBN * 2;          // state tile: 64 k-rows x 256 columns, four panels
constexpr int kAgStage = kAgA + kAgB;         // 48 KB
constexpr int kAgOffStage = kAgStages * kAgStage;
constexpr int kAgStaging = kAgBM * kAgBN * 2;  // 64 KB: four 64-column panels of 128 rows
constexpr int kAgOffBar = kAgOffStage + kAgStaging;
constexpr int kAgSmem = kAgOffBar + 256;

struct AggParams {
  float* zs;  // [B*H][nqb][d]
  int* status;
  int H, group, nqb, nk_steps, d;
  int m_tiles, n_tiles, tiles;  // tile t: m = m_first + t % m_tiles, n = (t / m_tiles) % n_tiles, bh = rest
  int m_first;                  // first row tile (a call that writes a range of query blocks)
};

__global__ void __launch_bounds__(kAgThreads, 1)
    aggregate_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmS, AggParams prm) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  volatile int* misc = reinterpret_cast<volatile int*>(smem + kAgOffBar + 128);  // tmem, abort
  auto bar = [&](int k) -> uint32_t { return sbase + kAgOffBar + 8 * k; };
  // ring full / empty per stage; accumulator full / empty per TMEM buffer
  constexpr int FULL = 0, EMPTY = kAgStages, ACC_FULL = 2 * kAgStages, ACC_EMPTY = ACC_FULL + 2;
  static_assert(ACC_EMPTY + 2 <= 16, "barrier area holds 16 mbarriers");
  if (tid == 0) {
    misc[1] = 0;
    for (int s = 0; s < kAgStages; ++s) {
      tc::mbar_init(bar(FULL + s), 1);
      tc::mbar_init(bar(EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(bar(ACC_FULL + a), 1);
      tc::mbar_init(bar(ACC_EMPTY + a), 4);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kAgOffBar + 128, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 1;
  const int K = prm.nk_steps;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = prm.tiles > (int)blockIdx.x ? (prm.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto tile_of = [&](int i, int& m0, int& n0, int& bh) {
    const int t = (int)blockIdx.x + i * (int)gridDim.x;
    m0 = (prm.m_first + t % prm.m_tiles) * kAgBM;
    n0 = ((t / prm.m_tiles) % prm.n_tiles) * kAgBN;
    bh = t / (prm.m_tiles * prm.n_tiles);
  };

  if (warp == 0) {
    // ======================= TMA producer =====================================
    if (lane == 0) {
      tc::prefetch_tensormap(&tmA);
      tc::prefetch_tensormap(&tmB);
      int kg = 0;  // ring use counter over all tiles
      for (int i = 0; i < my_tiles && !*abort; ++i) {
        int m0, n0, bh;
        tile_of(i, m0, n0, bh);
        const int bkv = (bh / prm.H) * (prm.H / prm.group) + (bh % prm.H) / prm.group;
        for (int k = 0; k < K; ++k, ++kg) {
          const int st = kg % kAgStages;
          if (kg >= kAgStages && !tc::mbar_wait(bar(EMPTY + st), ((kg / kAgStages) - 1) & 1, abort)) {
            *abort = 1;
            report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
            break;
          }
          const uint32_t a_s = sbase + st * kAgStage, b_s = a_s + kAgA;
          tc::mbar_expect_tx(bar(FULL + st), kAgStage);
          tc::tma_load_3d(a_s, &tmA, bar(FULL + st), k * 64, m0, bh);
          for (int p = 0; p < 4; ++p)
            tc::tma_load_3d(b_s + p * 8192, &tmB, bar(FULL + st), n0 + 64 * p, k * 64, bkv);
        }
      }
      // tail: every stage's last release has landed before the CTA exits
      for (int u = (kg > kAgStages ? kg - kAgStages : 0); u < kg && !*abort; ++u)
        if (!tc::mbar_wait(bar(EMPTY + u % kAgStages), (u / kAgStages) & 1, abort)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    constexpr uint32_t kId = tc::idesc_bf16(kAgBM, kAgBN, false, true);
    constexpr uint32_t kAll = 0xffffffffu;
    const uint64_t dA = tc::sw128_desc(sbase, 16, 1024);
    const uint64_t dB = tc::sw128_desc(sbase + kAgA, 8192, 1024);
    bool ok = true;
    int kg = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const int acc = i & 1, use = i >> 1;
      // the epilogue has read this accumulator's previous tile
      if (use > 0 && !__all_sync(kAll, tc::mbar_wait(bar(ACC_EMPTY + acc), (use - 1) & 1, abort))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      for (int k = 0; k < K; ++k, ++kg) {
        const int st = kg % kAgStages;
        if (!__all_sync(kAll, tc::mbar_wait(bar(FULL + st), (kg / kAgStages) & 1, abort))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t so = (uint32_t)(st * kAgStage) >> 4;
        if (tc::elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16_ss(tmem + acc * kAgBN, dA + so + (uint32_t)(kk * 32 >> 4),
                            dB + so + (uint32_t)(kk * 2048 >> 4), kId, (k > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(bar(EMPTY + st));
          if (k == K - 1) tc::mma_commit(bar(ACC_FULL + acc));
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else {
    // ======================= epilogue =========================================
    // thread = query block (TMEM lane) of the tile's 128 rows
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int dsq = prm.d * prm.d;
    const uint32_t stg = sbase + kAgOffStage;
    // Every epilogue warp runs both named barriers of every tile, also after a
    // failed wait (it then skips the work), so no warp is left at a barrier.
    bool ok = true;
    for (int i = 0; i < my_tiles; ++i) {
      int m0, n0, bh;
      tile_of(i, m0, n0, bh);
      const int acc = i & 1, use = i >> 1;
      ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(ACC_FULL + acc), use & 1, abort));
      tc::fence_after_sync();
      // the previous tile's TMA stores have finished reading the staging buffer
      if (r == 0) tc::bulk_wait_read_all();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const int row = m0 + r;
#pragma unroll 1
      for (int c64 = 0; c64 < kAgBN / 64 && ok; ++c64) {
        uint32_t v[2][32];
        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + acc * kAgBN + 64 * c64;
        tc::tmem_ld32(ta, v[0]);
        tc::tmem_ld32(ta + 32, v[1]);
        tc::tmem_ld_wait();
        const int col = n0 + 64 * c64;
        if (col < dsq) {
          uint4* srow = reinterpret_cast<uint4*>(smem + kAgOffStage + c64 * 16384 + r * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t* vv = v[q >> 2] + 8 * (q & 3);
            srow[q ^ (r & 7)] = make_uint4(pack_bf16(__uint_as_float(vv[0]), __uint_as_float(vv[1])),
                                           pack_bf16(__uint_as_float(vv[2]), __uint_as_float(vv[3])),
                                           pack_bf16(__uint_as_float(vv[4]), __uint_as_float(vv[5])),
                                           pack_bf16(__uint_as_float(vv[6]), __uint_as_float(vv[7])));
          }
        } else if (row < prm.nqb) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int cz = col + 32 * hf - dsq;
            if (cz >= prm.d) continue;
            float4* dst = reinterpret_cast<float4*>(prm.zs + ((size_t)bh * prm.nqb + row) * prm.d + cz);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(__uint_as_float(v[hf][4 * j]), __uint_as_float(v[hf][4 * j + 1]),
                                   __uint_as_float(v[hf][4 * j + 2]), __uint_as_float(v[hf][4 * j + 3]));
          }
        }
      }
      // the accumulator is read: the MMA warp may start the tile after next in it
      tc::fence_before_sync();
      __syncwarp();
      if (ok && lane == 0) tc::mbar_arrive(bar(ACC_EMPTY + acc));
      tc::fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (ok && r == 0 && m0 < prm.nqb) {
        // rows past nqb and columns past d*d fall outside the map and are not written
        for (int c64 = 0; c64 < kAgBN / 64; ++c64)
          if (n0 + 64 * c64 < dsq) tc::tma_store_3d(&tmS, stg + c64 * 16384, n0 + 64 * c64, m0, bh);
        tc::bulk_commit();
      }
    }
    if (r == 0) tc::bulk_wait_all();
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_aggregate(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const __nv_bfloat16* mm = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_mmask);
  const __nv_bfloat16* hs = reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_hs);
  CUtensorMap ma, mb;
  // mask [B*H][nqb_pad][nkb_pad], box 64 (k) x 128 (rows); states [B*H_kv][nkb_pad][dd], box 64 x 64
  if (!make_tmap_3d(&ma, mm, (uint64_t)p.nkb_pad, (uint64_t)p.nqb_pad, (uint64_t)c.B * c.H,
                    (uint64_t)p.nkb_pad * 2, (uint64_t)p.nqb_pad * p.nkb_pad * 2, 64, 128) ||
      !make_tmap_3d(&mb, hs, (uint64_t)p.dd, (uint64_t)p.nkb_pad, (uint64_t)c.B * c.H_kv,
                    (uint64_t)p.dd * 2, (uint64_t)p.nkb_pad * p.dd * 2, 64, 64))
    return cudaErrorInvalidValue;
  // S_i as [B*H][nqb rows][d*d columns], box 64 x 128 (stores)
  CUtensorMap ms;
  const uint64_t dsq = (uint64_t)c.d * c.d;
  if (!make_tmap_3d(&ms, a.ws + p.off_ss, dsq, (uint64_t)p.nqb, (uint64_t)c.B * c.H, dsq * 2,
                    (uint64_t)p.nqb * dsq * 2, 64, 128))
    return cudaErrorInvalidValue;
  AggParams prm;
  prm.zs = reinterpret_cast<float*>(a.ws + p.off_zs);
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.nqb = p.nqb;
  prm.nk_steps = p.nkb_pad / 64;
  prm.d = c.d;
  // the row tiles that hold the call's query blocks [qb0, qb1)
  prm.m_first = p.qb0 / kAgBM;
  prm.m_tiles = (p.qb1 + kAgBM - 1) / kAgBM - prm.m_first;
  prm.n_tiles = (p.dd + kAgBN - 1) / kAgBN;
  prm.tiles = prm.m_tiles * prm.n_tiles * c.B * c.H;
  cudaError_t e = cudaFuncSetAttribute(aggregate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kAgSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = prm.tiles < sms ? prm.tiles : sms;  // one persistent CTA per SM
  aggregate_tc_kernel<<<grid, kAgThreads, kAgSmem, s>>>(ma, mb, ms, prm);
  return cudaGetLastError();
}

}  // namespace sla

namespace sla {

// Backward: dh'_j = sum_i M[i, j] dS'_i and dz_j = sum_i M[i, j] dZ_i over the
// query blocks of every query head of the KV group, as the same GEMM with
//   A = M^T [B*H_kv][nkb_pad rows][group * nqb_pad]   (0/1, exact in bf16)
//   B = [dS'_i | dZ_i] rows [B*H_kv][group * nqb_pad][dd]
// and the output rows (key blocks) written to dh [B*H_kv][nkb][d*d] (bf16) and
// dz [B*H_kv][nkb][d] (fp32).
cudaError_t launch_aggregate_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const uint64_t bkv = (uint64_t)c.B * c.H_kv, rows_t = (uint64_t)bp.rows_t;
  CUtensorMap ma, mb, ms;
  if (!make_tmap_3d(&ma, a.bws + bp.off_maskt, rows_t, (uint64_t)p.nkb_pad, bkv, rows_t * 2,
                    (uint64_t)p.nkb_pad * rows_t * 2, 64, 128) ||
      !make_tmap_3d(&mb, a.bws + bp.off_drow, (uint64_t)p.dd, rows_t, bkv, (uint64_t)p.dd * 2, rows_t * p.dd * 2,
                    64, 64))
    return cudaErrorInvalidValue;
  const uint64_t dsq = (uint64_t)c.d * c.d;
  if (!make_tmap_3d(&ms, a.bws + bp.off_dh, dsq, (uint64_t)p.nkb, bkv, dsq * 2, (uint64_t)p.nkb * dsq * 2, 64, 128))
    return cudaErrorInvalidValue;
  AggParams prm;
  prm.zs = reinterpret_cast<float*>(a.bws + bp.off_dz);
  prm.status = a.status;
  prm.H = c.H_kv;  // one output "head" per KV head, reading its own right-hand side
  prm.group = 1;
  prm.nqb = p.nkb;
  prm.nk_steps = bp.rows_t / 64;
  prm.d = c.d;
  prm.m_first = 0;
  prm.m_tiles = (p.nkb + kAgBM - 1) / kAgBM;
  prm.n_tiles = (p.dd + kAgBN - 1) / kAgBN;
  prm.tiles = prm.m_tiles * prm.n_tiles * (int)bkv;
  cudaError_t e = cudaFuncSetAttribute(aggregate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kAgSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = prm.tiles < sms ? prm.tiles : sms;
  aggregate_tc_kernel<<<grid, kAgThreads, kAgSmem, s>>>(ma, mb, ms, prm);
  return cudaGetLastError();
}

}  // namespace sla
