// Aggregation of the linear branch on the 5th-generation tensor cores.
//
// For every query head, S_i = sum over the marginal blocks j of row i of the
// per-block state h_j (d x d, with W_p folded in) and Z_i = sum of z_j (SLA
// analysis page, arXiv 2509.24006: linear attention over the marginal blocks).
// Written as one GEMM per head:
//
//   C[i, :] = sum_j M[i, j] * Hs[j, :]     M: 0/1 marginal mask (exact in bf16)
//
// with C = [S_i | Z_i] row by row. One CTA computes a 256 (query blocks) x 256
// (state columns) tile as two M = 128 tcgen05 accumulators (all 512 TMEM
// columns), K = key blocks in steps of 64; A (the mask, K-major) and B (the
// states, N-major) come by TMA through a 3-stage ring. Large tiles keep the
// operand re-reads through L2 low: every state tile is read by nqb/256 CTAs,
// every mask tile by dd/256. The grid runs the query-block tiles of one column
// tile next to each other so a tile of states comes from HBM once.
//
// Warps: 0 = TMA producer, 1 = TMEM owner and MMA issuer, 2-5 = epilogue
// (S_i columns to bf16 staged for TMA stores, Z_i columns to fp32, padding
// columns dropped).
#include "common.cuh"
#include "tc.cuh"

namespace sla {

constexpr int kAgStages = 3;
constexpr int kAgThreads = 192;
constexpr int kAgBM = 256, kAgBN = 256;
constexpr int kAgA = kAgBM * 64 * 2;  // mask tile: 256 rows x 64 k, two 128-row boxes
constexpr int kAgB = 64 * kAgBN * 2;  // state tile: 64 k-rows x 256 columns, four panels
constexpr int kAgStage = kAgA + kAgB;
constexpr int kAgOffBar = kAgStages * kAgStage;
constexpr int kAgSmem = kAgOffBar + 128;

struct AggParams {
  __nv_bfloat16* ss;  // [B*H][nqb][d*d]
  float* zs;          // [B*H][nqb][d]
  int* status;
  int H, group, nqb, nk_steps, d;
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
  const int mt = blockIdx.x, nt = blockIdx.y, bh = blockIdx.z;
  const int m0 = mt * kAgBM, n0 = nt * kAgBN;
  const int b = bh / prm.H, h = bh % prm.H;
  const int bkv = b * (prm.H / prm.group) + h / prm.group;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + kAgOffBar + 64);  // tmem, abort
  auto bar = [&](int k) -> uint32_t { return sbase + kAgOffBar + 8 * k; };
  constexpr int FULL = 0, EMPTY = kAgStages, DONE = 2 * kAgStages;
  if (tid == 0) {
    misc[1] = 0;
    for (int s = 0; s < kAgStages; ++s) {
      tc::mbar_init(bar(FULL + s), 1);
      tc::mbar_init(bar(EMPTY + s), 1);
    }
    tc::mbar_init(bar(DONE), 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kAgOffBar + 64, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 1;
  const int K = prm.nk_steps;

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tensormap(&tmA);
      tc::prefetch_tensormap(&tmB);
      for (int k = 0; k < K; ++k) {
        const int st = k % kAgStages;
        if (k >= kAgStages && !tc::mbar_wait(bar(EMPTY + st), ((k / kAgStages) - 1) & 1, abort)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
          break;
        }
        const uint32_t a_s = sbase + st * kAgStage, b_s = a_s + kAgA;
        tc::mbar_expect_tx(bar(FULL + st), kAgStage);
        tc::tma_load_3d(a_s, &tmA, bar(FULL + st), k * 64, m0, bh);
        tc::tma_load_3d(a_s + 16384, &tmA, bar(FULL + st), k * 64, m0 + 128, bh);
        for (int p = 0; p < 4; ++p)
          tc::tma_load_3d(b_s + p * 8192, &tmB, bar(FULL + st), n0 + 64 * p, k * 64, bkv);
      }
      // tail: every stage's last release has landed before the CTA exits
      for (int k = (K > kAgStages ? K - kAgStages : 0); k < K && !*abort; ++k)
        if (!tc::mbar_wait(bar(EMPTY + k % kAgStages), (k / kAgStages) & 1, abort)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kId = tc::idesc_bf16(128, kAgBN, false, true);
      bool ok = true;
      for (int k = 0; k < K; ++k) {
        const int st = k % kAgStages;
        if (!tc::mbar_wait(bar(FULL + st), (k / kAgStages) & 1, abort)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t a_s = sbase + st * kAgStage, b_s = a_s + kAgA;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t db = tc::sw128_desc(b_s + kk * 2048, 8192, 1024);
#pragma unroll
          for (int mh = 0; mh < 2; ++mh) {
            const uint64_t da = tc::sw128_desc(a_s + mh * 16384 + kk * 32, 16, 1024);
            tc::mma_bf16_ss(tmem + mh * kAgBN, da, db, kId, (k > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(bar(EMPTY + st));
      }
      if (ok) tc::mma_commit(bar(DONE));
      if (!ok) {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    }
  } else {
    // epilogue: thread = query block (TMEM lane) of each 128-row half. S_i columns
    // are staged as bf16 in the freed stage ring (per half: four 64-column
    // panels of 128 rows, 128-byte swizzled) and written by TMA stores; Z_i
    // columns go straight to HBM as fp32.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, K > 0 && tc::mbar_wait(bar(DONE), 0, abort));
    tc::fence_after_sync();
    const int dsq = prm.d * prm.d;
    for (int mh = 0; mh < 2 && ok; ++mh) {
      const int row = m0 + mh * 128 + r;
#pragma unroll 1
      for (int c64 = 0; c64 < kAgBN / 64; ++c64) {
        uint32_t v[2][32];
        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + mh * kAgBN + 64 * c64;
        tc::tmem_ld32(ta, v[0]);
        tc::tmem_ld32(ta + 32, v[1]);
        tc::tmem_ld_wait();
        const int col = n0 + 64 * c64;
        if (col < dsq) {
          uint4* srow = reinterpret_cast<uint4*>(smem + mh * 65536 + c64 * 16384 + r * 128);
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
    }
    tc::fence_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok && quarter == 0 && lane == 0) {
      // rows past nqb and columns past d*d fall outside the map and are not written
      for (int mh = 0; mh < 2; ++mh)
        for (int c64 = 0; c64 < kAgBN / 64; ++c64)
          if (n0 + 64 * c64 < dsq && m0 + mh * 128 < prm.nqb)
            tc::tma_store_3d(&tmS, sbase + mh * 65536 + c64 * 16384, n0 + 64 * c64, m0 + mh * 128, bh);
      tc::bulk_commit();
      tc::bulk_wait_all();
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
  prm.ss = reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_ss);
  prm.zs = reinterpret_cast<float*>(a.ws + p.off_zs);
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.nqb = p.nqb;
  prm.nk_steps = p.nkb_pad / 64;
  prm.d = c.d;
  cudaError_t e = cudaFuncSetAttribute(aggregate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kAgSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nqb_pad + kAgBM - 1) / kAgBM, (p.dd + kAgBN - 1) / kAgBN, c.B * c.H);
  aggregate_tc_kernel<<<grid, kAgThreads, kAgSmem, s>>>(ma, mb, ms, prm);
  return cudaGetLastError();
}

}  // namespace sla
