// Backward pass of the sparse branch on the 5th-generation tensor cores.
//
// The sparse branch is exact softmax attention of each query block over the
// key tokens of its critical blocks (SLA analysis page, arXiv 2509.24006;
// 2025 sparse-attention review, section 2.3, NSA operator design: indexed KV
// blocks). Its gradient follows the FlashAttention recomputation: with the
// row log-sum-exp the forward kept (log2 domain, lse2_t), over every critical
// (query block i, key block j) tile
//   P = 2^(S * scale * log2 e - lse2),  S = Q_i K_j^T
//   dP = dO_i V_j^T,  dS = P * (dP - D_t),  D_t = dO_t . O_s,t
//   dQ_i += scale dS K_j,  dK_j += scale dS^T Q_i,  dV_j += P^T dO_i
// Two kernels, each with one writer per output row (no atomics):
//   flash_dq_kernel    128 query rows (blocks 2p, 2p+1 of a head), their merged
//                      critical key blocks streamed through a ring;
//   flash_dkdv_kernel  128 key rows (blocks 2p, 2p+1 of a KV head), for every
//                      query head of the group the query blocks that hold
//                      either key block as critical, streamed through a ring.
// The query blocks of a key block come from a bitmap per (head, key block)
// that cols_mark_kernel fills from the critical lists.
// Warps 0-7: two warpgroups, one TMEM lane quarter per warp (thread = row),
// the warpgroups taking the two 32-column halves of every tile; warps 8 and 10:
// tcgen05.mma issue (one elected lane each: the S / dP products, the dQ / dV / dK
// products); warp 9: TMA loads into a ring of four or five slots, refilled as soon as a
// slot frees; warp 11: the unit loader. The row warps write P and dS back into TMEM
// as bf16 pairs and the dQ / dV / dK products read them from there (A operand in TMEM).
// Both kernels are persistent (one CTA per SM, units from a counter): the loader builds
// the next unit's list and loads its stationary tiles while the current unit runs, the
// ring runs on across units, and the next unit's products start during the current
// unit's epilogue. Both add the linear-branch part of the gradient (fp32 scratch) and
// write the final bf16 rows.
#include <cstring>

#include "common.cuh"
#include "tc.cuh"

namespace sla {

// ---------------------------------------------------------------------------
// column bitmaps: bit i of bits[row][j] is set when query block i has key block j
// critical (three-way: row = query head) or selected (top-n: row = KV head; the
// selection is shared by the group, -1 entries are padding)
// ---------------------------------------------------------------------------
__global__ void cols_mark_kernel(const int32_t* __restrict__ crit, uint32_t* __restrict__ bits, int64_t entries,
                                 int nqb, int nkb, int len, int words, int topn, int* status) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < entries; e += stride) {
    const int64_t row = e / len;  // (head or KV head) * nqb + i
    const int hr = (int)(row / nqb), i = (int)(row % nqb);
    const int j = crit[e];
    if (topn && j < 0) continue;
    if (j < 0 || j >= nkb || (topn && j >= i)) {
      report(status, SLA_ERR_DEVICE_CHECK, kDetailFlashIndex);
      continue;
    }
    atomicOr(bits + ((size_t)hr * nkb + j) * words + (i >> 5), 1u << (i & 31));
  }
}

cudaError_t launch_cols(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const bool topn = c.mode == SLA_MODE_TOPN_WINDOW;
  const int rows = topn ? c.H_kv : c.H, len = topn ? c.top_n : c.k_h;
  uint32_t* bits = reinterpret_cast<uint32_t*>(a.bws + bp.off_bits);
  cudaError_t e = cudaMemsetAsync(bits, 0, (size_t)c.B * rows * p.nkb * bp.words * 4, s);
  if (e != cudaSuccess || len == 0) return e;
  const int64_t entries = (int64_t)c.B * rows * p.nqb * len;
  int64_t blocks = (entries + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  cols_mark_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const int32_t*>(a.ws + p.off_crit), bits,
                                                    entries, p.nqb, p.nkb, len, bp.words, topn ? 1 : 0, a.status);
  return cudaGetLastError();
}

// Kernel modes. kModeNsa (dQ) and kModeNsaTok / kModeNsaCmp (dK, dV) are NSA's three
// branches (sparse attention survey, section 2: compressed, selected and window
// attention, each its own softmax, summed with gates). Each branch b has its own row
// log-sum-exp and D values; the gate is folded into the log-sum-exp (lse_b - log2 g_b),
// so that the recomputed P is g_b P_b and dS = g_b P_b (dP - D_b) with D_b = dO . o_b:
// the gradient of g_b o_b with the unscaled dO.
constexpr int kModeThree = 0, kModeTopn = 1, kModeNsa = 2, kModeNsaTok = 2, kModeNsaCmp = 3;
enum NsaBranch { kBrCmp = 0, kBrSel = 1, kBrWin = 2 };

// warps 0-7: rows (two column halves); warp 8: TMEM owner and issuer of the S / dP
// (S^T / dP^T) products; warp 9: TMA producer of the streamed tiles; warp 10: issuer of the
// dQ (dV, dK) products; warp 11: unit loader (the next unit's list and stationary tiles).
// Two issuer warps, so that one warp's barrier waits (about 160 cycles each, measured) do
// not leave the tensor pipe without queued work.
constexpr int kMmaWarp = 8, kProdWarp = 9, kRowWarps = 8, kDqWarp = 10, kLoadWarp = 11;
constexpr int kBwThreads = 384;
constexpr int kListReaders = kRowWarps + 3;  // warps that arrive on a unit's LIST_FREE
// The loader takes the next unit when the producer has this many tiles of the current one
// left to load (at once for shorter units): time to build the list and load the stationary
// tiles, without committing a long unit to a CTA long before it can start.
constexpr int kClaimLead = 64;

// merged list of two bitmaps (warp 0, ascending). Entry = index (bits 0-12) | a0 << 13 | a1 << 14
// | s0 << 15 | s1 << 16 | tag << 17: a0 / a1 = the index is in bitmap a0 / a1 ("active" for
// half 0 / 1), s0 / s1 = in bitmap s0 / s1 (top-n mode: "selected", NULL elsewhere).
// Returns the count (in every lane).
constexpr uint32_t kIdxMask = 0x1FFFu;
constexpr int kActBit = 13, kSelBit = 15, kTagShift = 17;
__device__ __forceinline__ int merge_bitmaps(const uint32_t* a0p, const uint32_t* a1p, const uint32_t* s0p,
                                             const uint32_t* s1p, int words, bool v0, bool v1, uint32_t tag,
                                             uint32_t* out, int base, int lane) {
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t a0 = (w < words && v0) ? a0p[w] : 0u, a1 = (w < words && v1) ? a1p[w] : 0u;
    const uint32_t s0 = (s0p && w < words && v0) ? s0p[w] : 0u, s1 = (s1p && w < words && v1) ? s1p[w] : 0u;
    uint32_t any = a0 | a1;
    const int cnt = __popc(any);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - cnt;
    while (any) {
      const int bit = __ffs(any) - 1;
      any &= any - 1;
      const uint32_t m = 1u << bit;
      out[pos++] = (uint32_t)(w * 32 + bit) | ((a0 & m) ? 1u << kActBit : 0u) | ((a1 & m) ? 1u << (kActBit + 1) : 0u) |
                   ((s0 & m) ? 1u << kSelBit : 0u) | ((s1 & m) ? 1u << (kSelBit + 1) : 0u) | (tag << kTagShift);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  return base;
}

// 32 consecutive floats of a row (chunk ch: columns 32 ch .. 32 ch + 31), zeros without a row
__device__ __forceinline__ void load_row32(const float* row, int ch, float4 (&a)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    a[j] = row ? *reinterpret_cast<const float4*>(row + 32 * ch + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
template <int D, int SL>  // SL ring slots
struct DqLayout {
  static constexpr int NP = D / 64;
  static constexpr int kOffQ = 0;                         // Q: 128 rows, NP panels of 16 KB
  static constexpr int kOffO = kOffQ + NP * 16384;        // dO
  static constexpr int kTile = NP * 8192;                 // one 64-row K or V tile
  static constexpr int kSlot = 2 * kTile;                 // K_j, V_j
  static constexpr int kOffRing = kOffO + NP * 16384;
  static constexpr int kOffBar = kOffRing + SL * kSlot;  // 32 mbarriers
  static constexpr int kOffMisc = kOffBar + 32 * 8;      // TMEM address, abort flag, two unit headers
  static constexpr int kOffList = kOffMisc + 64;          // two merged block lists, then the loader's bitmaps
  static constexpr int kTmemCols = 512;                   // dQ: D; S / dP: 2 x 128; dS: 2 x 32; Q: D / 2
  static constexpr int kQCol = D + 320;                   // Q as the A operand of S = Q K^T (bf16 pairs)
  static_assert(kQCol + D / 2 <= kTmemCols, "TMEM columns");
};

struct DqParams {
  const int32_t* crit;   // three-way: [B*H][nqb][len] critical; top-n: [B*H_kv][nqb][len] selected (-1 pad)
  const float* lse;      // [B*H][N] (log2 domain); NSA: [3][B*H][N] per branch, gate folded in
  const float* delta;    // [B*H][N]; NSA: [3][B*H][N]
  const float* dq_acc;   // [B*H][N][D] or null
  __nv_bfloat16* dq;     // [B*H][N][D]
  int* status;
  int* counter;          // units handed out so far (0 at launch)
  int H, group, N, n_valid, nb, len, npairs, words, window, units, list_cap;
  float scale, scale_log2;
  // NSA: branch stride of lse / delta / dlogit (B*H*N), the gate logits' gradients
  // dlogit [3][B*H][N] and gates w_g [H][3][D] (both null without gates), the compressed
  // keys (n_cmp keys in nct 64-key tiles, key c stands for token c * kstride + kspan)
  size_t bstride;
  const float* dlogit;
  const __nv_bfloat16* w_g3;
  int n_cmp, nct, kstride, kspan;
};

// The merged key-block list of one dQ unit (query blocks 2 pr, 2 pr + 1 of head bh), built
// by one warp from the routing's lists through four bitmaps (active blocks of half 0 / 1,
// selected blocks of half 0 / 1) in `words`. Returns the count (in every lane).
template <bool TOPN, bool NSA>
__device__ int dq_unit_list(const DqParams& prm, int bh, int bkv, int pr, uint32_t* words, uint32_t* mlist,
                            int lane) {
  const int i_h[2] = {2 * pr, 2 * pr + 1};
  const bool valid_h[2] = {i_h[0] < prm.nb, i_h[1] < prm.nb};
  for (int w = lane; w < 4 * prm.words; w += 32) words[w] = 0u;
  __syncwarp();
  for (int hf = 0; hf < 2; ++hf) {
    if (!valid_h[hf]) continue;
    const int32_t* lst = prm.crit + ((size_t)(TOPN ? bkv : bh) * prm.nb + i_h[hf]) * prm.len;
    uint32_t* act = words + hf * prm.words;
    uint32_t* sel = words + (2 + hf) * prm.words;
    for (int e = lane; e < prm.len; e += 32) {
      const int j = lst[e];
      if (TOPN && j < 0) continue;  // padding of short selections
      if (j < 0 || j >= prm.nb || (TOPN && j >= i_h[hf])) {
        report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashIndex);
        continue;
      }
      if (!NSA) atomicOr(&act[j >> 5], 1u << (j & 31));  // NSA: act holds the window alone
      if (TOPN) atomicOr(&sel[j >> 5], 1u << (j & 31));
    }
    if (TOPN && prm.window > 0) {  // the blocks the causal window reaches
      const int lo = i_h[hf] * kBlock - prm.window + 1;
      const int first = lo <= 0 ? 0 : lo / kBlock;
      for (int j = first + lane; j <= i_h[hf]; j += 32) atomicOr(&act[j >> 5], 1u << (j & 31));
    }
  }
  __syncwarp();
  int n = 0;
  if (NSA) {
    // compressed key tiles up to the causal limit of either half (act bit per half),
    // then the selected blocks, then the window blocks; the tag is the branch
    int jmax[2];
    for (int hf = 0; hf < 2; ++hf) {
      const int last_t = i_h[hf] * kBlock + kBlock - 1 - prm.kspan;
      int jm = (!valid_h[hf] || last_t < 0 || prm.n_cmp == 0) ? -1 : last_t / prm.kstride / kBlock;
      const int jcap = (prm.n_cmp - 1) / kBlock;
      jmax[hf] = jm > jcap ? jcap : jm;
    }
    const int nc = (jmax[0] > jmax[1] ? jmax[0] : jmax[1]) + 1;
    for (int jt = lane; jt < nc; jt += 32)
      mlist[jt] = (uint32_t)jt | (jt <= jmax[0] ? 1u << kActBit : 0u) | (jt <= jmax[1] ? 1u << (kActBit + 1) : 0u) |
                  ((uint32_t)kBrCmp << kTagShift);
    __syncwarp();
    n = merge_bitmaps(words + 2 * prm.words, words + 3 * prm.words, words + 2 * prm.words, words + 3 * prm.words,
                      prm.words, true, true, (uint32_t)kBrSel, mlist, nc > 0 ? nc : 0, lane);
    n = merge_bitmaps(words, words + prm.words, nullptr, nullptr, prm.words, true, true, (uint32_t)kBrWin, mlist, n,
                      lane);
  } else {
    n = merge_bitmaps(words, words + prm.words, TOPN ? words + 2 * prm.words : nullptr,
                      TOPN ? words + 3 * prm.words : nullptr, prm.words, true, true, 0u, mlist, 0, lane);
  }
  __syncwarp();
  return n;
}

// TOPN: element (t, s) is kept when s <= t and (block(s) selected or s > t - window).
// NSA: the list holds three kinds of tiles, tagged with their branch: compressed key tiles
// (tmKc / tmVc; key c kept when c < n_cmp and c * kstride + kspan <= t), selected blocks
// (s <= t) and window blocks (t - window < s <= t). All of them add to one dQ accumulator.
// Persistent: one CTA per SM takes units (pairs of query blocks) from prm.counter.
template <int D, int MODE, int SL>
__global__ void __launch_bounds__(kBwThreads, 1)
    flash_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                    DqParams prm) {
  constexpr bool TOPN = MODE != kModeThree, NSA = MODE == kModeNsa;
  using L = DqLayout<D, SL>;
  constexpr int NP = L::NP, S = SL;
  constexpr uint32_t kAll = 0xffffffffu;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);  // tmem, -, abort, -, headers
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + L::kOffList);
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  // header of this CTA's unit u: the unit index (-1: no more units) and its tile count
  auto hdr = [&](int u) { return misc + 4 + 2 * (u & 1); };
  auto unit_list = [&](int u) { return lists + (u & 1) * prm.list_cap; };
  auto kv_head = [&](int bh) { return (bh / prm.H) * (prm.H / prm.group) + (bh % prm.H) / prm.group; };
  // ring slots: LOADED (K_j, V_j landed), SLOT_FREE (the dQ product read them); S / dP
  // buffers: SP_FULL (products done), S_READ (row warps have loaded them); dS buffers:
  // DS_FULL (written), DS_FREE (dQ product done). Per unit: LIST_FULL / LIST_FREE (its
  // header and list, two buffers), Q_FULL / DO_FULL (Q, dO landed), Q_TMEM (row warps have
  // copied Q into TMEM), PROD_DONE (its S / dP products are done: dO and the Q columns may
  // be overwritten), ACC_DONE (its dQ is complete), ACC_FREE (row warps have read dQ)
  constexpr int LOADED = 0, SLOT_FREE = S, SP_FULL = 2 * S, S_READ = SP_FULL + 2, DS_FULL = S_READ + 2,
                DS_FREE = DS_FULL + 2, LIST_FULL = DS_FREE + 2, LIST_FREE = LIST_FULL + 2, Q_FULL = LIST_FREE + 2,
                DO_FULL = Q_FULL + 1, Q_TMEM = DO_FULL + 1, PROD_DONE = Q_TMEM + 1, ACC_DONE = PROD_DONE + 1,
                ACC_FREE = ACC_DONE + 1, CLAIM = ACC_FREE + 1;
  static_assert(CLAIM < 32, "mbarriers");
  if (tid == 0) {
    misc[2] = 0;
    for (int x = 0; x < S; ++x) {
      tc::mbar_init(bar(LOADED + x), 1);
      tc::mbar_init(bar(SLOT_FREE + x), 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar(SP_FULL + x), 1);
      tc::mbar_init(bar(S_READ + x), kRowWarps);
      tc::mbar_init(bar(DS_FULL + x), kRowWarps);
      tc::mbar_init(bar(DS_FREE + x), 1);
      tc::mbar_init(bar(LIST_FULL + x), 1);
      tc::mbar_init(bar(LIST_FREE + x), kListReaders);
    }
    tc::mbar_init(bar(Q_FULL), 1);
    tc::mbar_init(bar(DO_FULL), 1);
    tc::mbar_init(bar(Q_TMEM), kRowWarps);
    tc::mbar_init(bar(PROD_DONE), 1);
    tc::mbar_init(bar(ACC_DONE), 1);
    tc::mbar_init(bar(ACC_FREE), kRowWarps);
    tc::mbar_init(bar(CLAIM), 1);
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(sbase + L::kOffMisc, L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 2;
  const uint32_t sQ = sbase + L::kOffQ, sO = sbase + L::kOffO, sR = sbase + L::kOffRing;
  bool ok = true;

  if (warp == kLoadWarp) {
    // ======================= unit loader ======================================
    // the next unit's list, then its Q (once the row warps have copied the previous Q into
    // TMEM) and dO (once the previous unit's products are done); every unit takes these
    // steps, with or without tiles
    uint32_t* words = lists + 2 * prm.list_cap;
    int prev = -1;
    for (int u = 0;; ++u) {
      // the next unit is taken once the producer is within kClaimLead tiles of the current
      // unit's end: a unit is committed to this CTA only shortly before it can start
      if (u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(CLAIM), (u - 1) & 1, abort));
      if (!ok) break;
      int x = 0;
      if (lane == 0) x = atomicAdd(prm.counter, 1);
      x = __shfl_sync(kAll, x, 0);
      if (u >= 2) ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FREE + (u & 1)), ((u - 2) >> 1) & 1, abort));
      if (!ok) break;
      volatile int* h = hdr(u);
      if (x >= prm.units) {
        if (lane == 0) {
          h[0] = -1;
          h[1] = 0;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(LIST_FULL + (u & 1)));
        break;
      }
      const int bh = x / prm.npairs, pr = x % prm.npairs;
      const int n = dq_unit_list<TOPN, NSA>(prm, bh, kv_head(bh), pr, words, unit_list(u), lane);
      if (lane == 0) {
        h[0] = x;
        h[1] = n;
      }
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(bar(LIST_FULL + (u & 1)));
        if (u >= 1) ok = tc::mbar_wait(bar(Q_TMEM), (u - 1) & 1, abort);
        if (ok) {
          tc::mbar_expect_tx(bar(Q_FULL), 2 * NP * 8192);
          for (int hf = 0; hf < 2; ++hf)
            for (int p = 0; p < NP; ++p)
              tc::tma_load_3d(sQ + p * 16384 + hf * 8192, &tmQ, bar(Q_FULL), 64 * p, (2 * pr + hf) * kBlock, bh);
        }
        if (ok && u >= 1) ok = tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort);
        if (ok) {
          tc::mbar_expect_tx(bar(DO_FULL), 2 * NP * 8192);
          for (int hf = 0; hf < 2; ++hf)
            for (int p = 0; p < NP; ++p)
              tc::tma_load_3d(sO + p * 16384 + hf * 8192, &tmO, bar(DO_FULL), 64 * p, (2 * pr + hf) * kBlock, bh);
          // the previous unit's epilogue reads its linear part next: into L2 ahead of it
          if (prev >= 0 && prm.dq_acc != nullptr) {
            const int t0 = 2 * (prev % prm.npairs) * kBlock;
            const int rows = prm.N - t0 < 2 * kBlock ? prm.N - t0 : 2 * kBlock;
            tc::prefetch_l2(prm.dq_acc + ((size_t)(prev / prm.npairs) * prm.N + t0) * D, (uint32_t)rows * D * 4);
          }
        }
      }
      ok = __shfl_sync(kAll, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      prev = x;
    }
    if (ok && lane == 0 && prev >= 0 && prm.dq_acc != nullptr) {  // the last unit's linear part
      const int t0 = 2 * (prev % prm.npairs) * kBlock;
      const int rows = prm.N - t0 < 2 * kBlock ? prm.N - t0 : 2 * kBlock;
      tc::prefetch_l2(prm.dq_acc + ((size_t)(prev / prm.npairs) * prm.N + t0) * D, (uint32_t)rows * D * 4);
    }
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp == kProdWarp) {
    // ======================= TMA producer: the K / V ring, across units ========
    if (lane == 0) {
      int g = 0;  // tiles of this CTA so far
      for (int u = 0;; ++u) {
        if (!(ok = tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort))) break;
        const int x = hdr(u)[0], T = hdr(u)[1];
        if (x < 0) break;
        const uint32_t* ml = unit_list(u);
        const int bkv = kv_head(x / prm.npairs);
        const int claim_at = T > kClaimLead ? T - kClaimLead : 0;
        if (claim_at == 0) tc::mbar_arrive(bar(CLAIM));
        for (int m = 0; m < T && ok; ++m, ++g) {
          if (m == claim_at && m > 0) tc::mbar_arrive(bar(CLAIM));
          const int slot = g % S;
          if (g >= S && !(ok = tc::mbar_wait(bar(SLOT_FREE + slot), ((g / S) - 1) & 1, abort))) break;
          const uint32_t e = ml[m];
          const int jb = (int)(e & kIdxMask);
          const bool cmp_tile = NSA && (e >> kTagShift) == (uint32_t)kBrCmp;
          const CUtensorMap* mk = cmp_tile ? &tmKc : &tmK;
          const CUtensorMap* mv = cmp_tile ? &tmVc : &tmV;
          const uint32_t dst = sR + slot * L::kSlot;
          tc::mbar_expect_tx(bar(LOADED + slot), L::kSlot);
          for (int p = 0; p < NP; ++p) {
            tc::tma_load_3d(dst + p * 8192, mk, bar(LOADED + slot), 64 * p, jb * kBlock, bkv);
            tc::tma_load_3d(dst + L::kTile + p * 8192, mv, bar(LOADED + slot), 64 * p, jb * kBlock, bkv);
          }
        }
        tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      }
      // the last release of every slot: no product reads the ring and no commit is in flight at exit
      for (int m = (g > S ? g - S : 0); m < g && ok; ++m)
        ok = tc::mbar_wait(bar(SLOT_FREE + m % S), (m / S) & 1, abort);
      if (!ok) {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= S / dP issuer ====================================
    constexpr uint32_t kIdS = tc::idesc_bf16(128, 64, false, false);
    // base descriptors; a byte offset off is added as off >> 4 (start-address field)
    const uint64_t dOd = tc::sw128_desc(sO, 16, 1024);
    const uint64_t dRk = tc::sw128_desc(sR, 16, 1024);    // ring tiles, K-major
    // S_g = Q K_g^T (A = Q in TMEM: only K is read from shared memory, full rate at N = 64)
    // and dP_g = dO V_g^T into TMEM buffer g & 1
    auto issue_sp = [&](int g) {
      const uint32_t so = (uint32_t)((g % S) * L::kSlot);
      const uint32_t tS = tmem + D + 128 * (g & 1);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t qo = (uint32_t)((k >> 2) * 16384 + (k & 3) * 32), ko = (uint32_t)((k >> 2) * 8192 + (k & 3) * 32);
        tc::mma_bf16_ts(tS, tmem + L::kQCol + 8 * k, dRk + ((so + ko) >> 4), kIdS, k > 0);
        tc::mma_bf16_ss(tS + 64, dOd + (qo >> 4), dRk + ((so + L::kTile + ko) >> 4), kIdS, k > 0);
      }
      tc::mma_commit(bar(SP_FULL + (g & 1)));
    };
    int g = 0, u = 0;
    for (;; ++u) {
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort)))) break;
      const int x = hdr(u)[0], T = hdr(u)[1];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (x < 0) break;
      ok = __all_sync(kAll, tc::mbar_wait(bar(Q_TMEM), u & 1, abort)) &&
           __all_sync(kAll, tc::mbar_wait(bar(DO_FULL), u & 1, abort));
      if (!ok) break;
      tc::fence_after_sync();
      for (int m = 0; m < T && ok; ++m, ++g) {
        // S / dP buffer g & 1 is free as soon as the row warps have loaded S_{g-2}, dP_{g-2}:
        // the products of tile g run while they compute dS_{g-2}
        if (g >= 2) ok = __all_sync(kAll, tc::mbar_wait(bar(S_READ + (g & 1)), ((g - 2) >> 1) & 1, abort));
        ok = ok && __all_sync(kAll, tc::mbar_wait(bar(LOADED + g % S), (g / S) & 1, abort));
        tc::fence_after_sync();
        if (ok && tc::elect_one()) {
          issue_sp(g);
          if (m == T - 1) tc::mma_commit(bar(PROD_DONE));
        }
        __syncwarp();
      }
      if (ok && T == 0 && tc::elect_one()) tc::mma_commit(bar(PROD_DONE));
      __syncwarp();
      if (!ok) break;
    }
    // the last unit's PROD_DONE has landed before the CTA exits
    if (ok && u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort));
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp == kDqWarp) {
    // ======================= dQ issuer =========================================
    constexpr uint32_t kIdQ = tc::idesc_bf16(128, D, false, true);
    const uint64_t dRn = tc::sw128_desc(sR, 8192, 1024);  // ring tiles, N-major (64-row panels)
    int g = 0, u = 0;
    for (;; ++u) {
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort)))) break;
      const int x = hdr(u)[0], T = hdr(u)[1];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (x < 0) break;
      // the accumulator is free once the row warps have read the previous unit's dQ
      if (u >= 1 && !(ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_FREE), (u - 1) & 1, abort)))) break;
      for (int m = 0; m < T && ok; ++m, ++g) {
        const int b = g & 1;
        if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(DS_FULL + b), (g >> 1) & 1, abort)))) break;
        tc::fence_after_sync();
        if (tc::elect_one()) {
          // dQ += dS_g K_g: A = dS_g from its TMEM buffer (bf16 pairs), B = K_g N-major. The
          // slot is released after this product: S_g, dP_g (its other readers) completed
          // before the row warps could write dS_g
          const uint32_t so = (uint32_t)((g % S) * L::kSlot);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16_ts(tmem, tmem + D + 256 + 32 * b + 8 * kk, dRn + ((so + kk * 2048) >> 4), kIdQ,
                            (m > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(bar(SLOT_FREE + g % S));
          tc::mma_commit(bar(DS_FREE + b));
          if (m == T - 1) tc::mma_commit(bar(ACC_DONE));
        }
        __syncwarp();
      }
      if (ok && T == 0 && tc::elect_one()) tc::mma_commit(bar(ACC_DONE));
      __syncwarp();
      if (!ok) break;
    }
    // the last two dS buffers' releases and the last ACC_DONE: no commit is in flight at exit
    for (int m = (g > 2 ? g - 2 : 0); m < g && ok; ++m)
      ok = __all_sync(kAll, tc::mbar_wait(bar(DS_FREE + (m & 1)), (m >> 1) & 1, abort));
    if (ok && u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_DONE), (u - 1) & 1, abort));
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp < kRowWarps) {
    // ======================= rows: dS, then the dq epilogue ===================
    // warp = quarter (TMEM lanes) + 4 * hw (key columns 32 hw .. 32 hw + 31 of each tile)
    const int quarter = warp & 3, hw = warp >> 2;
    const int r = quarter * 32 + lane, hf = r >> 6;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = prm.scale_log2;
    // Q row r (the TMEM lane) into columns kQCol.. as bf16 pairs, this warpgroup's half of the
    // features, from the swizzled Q tile (16-byte chunk c of a row at c ^ (row & 7)), once
    // unit u's Q has landed and the previous unit's S products are done
    auto copy_q = [&](int u) {
      bool fine = true;
      if (u >= 1) fine = __all_sync(kAll, tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort));
      fine = fine && __all_sync(kAll, tc::mbar_wait(bar(Q_FULL), u & 1, abort));
      if (fine) {
        tc::fence_after_sync();
        constexpr int CH = D / 16;  // 16-byte chunks per warpgroup half: 8 (D = 128) or 4
        uint32_t qv[CH * 4];
#pragma unroll
        for (int x = 0; x < CH; ++x) {
          const int chunk = hw * CH + x;  // of the row's D / 8 chunks
          const int p = chunk >> 3, c = chunk & 7;
          const uint4 v4 = *reinterpret_cast<const uint4*>(smem + L::kOffQ + p * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
          qv[4 * x] = v4.x; qv[4 * x + 1] = v4.y; qv[4 * x + 2] = v4.z; qv[4 * x + 3] = v4.w;
        }
        if constexpr (CH * 4 == 32)
          tc::tmem_st32(tmem + lane_off + L::kQCol + 32 * hw, *reinterpret_cast<const uint32_t(*)[32]>(qv));
        else
          tc::tmem_st16(tmem + lane_off + L::kQCol + 16 * hw, *reinterpret_cast<const uint32_t(*)[16]>(qv));
        tc::tmem_st_wait();
      }
      tc::fence_async_smem();  // the Q tile's reads come before the next unit's load into it
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(Q_TMEM));
      return fine;
    };
    // this row's log-sum-exp and D of unit x, per branch (NSA: compressed, selected, window;
    // otherwise one), read one unit ahead
    float lse_n[NSA ? 3 : 1], dlt_n[NSA ? 3 : 1];
    auto load_ld = [&](int x) {
      const int bh = x / prm.npairs, ih = 2 * (x % prm.npairs) + hf, t = ih * kBlock + (r & 63);
      const bool vrow = x >= 0 && ih < prm.nb && t < prm.n_valid;
#pragma unroll
      for (int x2 = 0; x2 < (NSA ? 3 : 1); ++x2) {
        lse_n[x2] = vrow ? prm.lse[x2 * prm.bstride + (size_t)bh * prm.N + t] : INFINITY;
        dlt_n[x2] = vrow ? prm.delta[x2 * prm.bstride + (size_t)bh * prm.N + t] : 0.f;
      }
    };
    int g = 0;
    ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL), 0, abort));
    if (ok && hdr(0)[0] >= 0) {
      load_ld(hdr(0)[0]);
      ok = copy_q(0);
    }
    for (int u = 0; ok; ++u) {
      const int x = hdr(u)[0], T = hdr(u)[1];
      if (x < 0) break;
      const uint32_t* ml = unit_list(u);
      const int bh = x / prm.npairs, pr = x % prm.npairs;
      const int ih = 2 * pr + hf;  // this row's query block
      const bool valid = ih < prm.nb;
      const int t = ih * kBlock + (r & 63);
      const int t_w = ih * kBlock + ((quarter * 32) & 63);  // first row of this warp
      const bool vrow = valid && t < prm.n_valid;
      float lse_b[NSA ? 3 : 1], dlt_b[NSA ? 3 : 1];
#pragma unroll
      for (int x2 = 0; x2 < (NSA ? 3 : 1); ++x2) {
        lse_b[x2] = lse_n[x2];
        dlt_b[x2] = dlt_n[x2];
      }
      for (int m = 0; m < T && ok; ++m, ++g) {
        const int b = g & 1;
        const uint32_t e = ml[m];
        const int k0 = (int)(e & kIdxMask) * kBlock;
        const bool act = (e >> (kActBit + hf)) & 1u;
        const bool sel = (e >> (kSelBit + hf)) & 1u;
        const int br = NSA ? (int)(e >> kTagShift) : 0;
        const bool cmp_tile = NSA && br == kBrCmp;
        const float lse2 = NSA ? (br == kBrCmp ? lse_b[0] : br == kBrSel ? lse_b[1] : lse_b[2]) : lse_b[0];
        const float dlt = NSA ? (br == kBrCmp ? dlt_b[0] : br == kBrSel ? dlt_b[1] : dlt_b[2]) : dlt_b[0];
        if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(SP_FULL + b), (g >> 1) & 1, abort)))) break;
        tc::fence_after_sync();
        const uint32_t tS = tmem + lane_off + D + 128 * b;
        uint32_t sv[32], pv[32];
        tc::tmem_ld32(tS + 32 * hw, sv);
        tc::tmem_ld32(tS + 64 + 32 * hw, pv);
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(S_READ + b));
        const int kc = k0 + 32 * hw;  // first key of this half
        // warp-uniform: every (row, key) of this warp's 32 x 32 sub-tile is kept, so no
        // per-element mask (rows t_w .. t_w + 31, keys kc .. kc + 31)
        bool full;
        if (cmp_tile)
          full = kc + 31 < prm.n_cmp && (kc + 31) * prm.kstride + prm.kspan <= t_w;
        else {
          full = kc + 31 < prm.n_valid;
          if (TOPN) full = full && kc + 31 <= t_w && (sel || kc > t_w + 31 - prm.window);
        }
        full = full && act;
        // P = 2^(s * scale * log2 e - lse), dS = P (dP - D), two columns per packed op
        const uint64_t sc2 = tc::f2_pack(sl2, sl2), nl2 = tc::f2_pack(-lse2, -lse2), dl2 = tc::f2_pack(dlt, dlt);
        uint32_t ds[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) ds[j] = 0u;  // a half that does not use the tile
        if (act)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint64_t y = tc::ffma2(tc::f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), sc2, nl2);
          float p0 = tc::ex2_approx(tc::f2_lo(y)), p1 = tc::ex2_approx(tc::f2_hi(y));
          if (!full) {
            bool keep[2];
#pragma unroll
            for (int x2 = 0; x2 < 2; ++x2) {
              const int key = kc + 2 * j + x2;
              if (cmp_tile)
                keep[x2] = act && key < prm.n_cmp && key * prm.kstride + prm.kspan <= t;
              else {
                keep[x2] = act && key < prm.n_valid;
                if (TOPN) keep[x2] = keep[x2] && key <= t && (sel || key > t - prm.window);
              }
            }
            p0 = keep[0] ? p0 : 0.f;
            p1 = keep[1] ? p1 : 0.f;
          }
          const uint64_t gg = tc::fmul2(tc::f2_pack(p0, p1),
                                        tc::fsub2(tc::f2_pack(__uint_as_float(pv[2 * j]), __uint_as_float(pv[2 * j + 1])), dl2));
          ds[j] = pack_bf16(tc::f2_lo(gg), tc::f2_hi(gg));
        }
        // dS buffer b was last read by the dQ product of tile g - 2
        if (g >= 2 && !(ok = __all_sync(kAll, tc::mbar_wait(bar(DS_FREE + b), ((g - 2) >> 1) & 1, abort)))) break;
        tc::fence_after_sync();
        tc::tmem_st16(tmem + lane_off + D + 256 + 32 * b + 16 * hw, ds);
        tc::tmem_st_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(DS_FULL + b));
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (!ok) break;
      // the next unit's Q into TMEM before this unit's epilogue, so that its first products
      // run meanwhile
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + ((u + 1) & 1)), ((u + 1) >> 1) & 1, abort)))) break;
      const int x_next = hdr(u + 1)[0];
      const bool more = x_next >= 0;
      if (more) load_ld(x_next);
      if (more && !(ok = copy_q(u + 1))) break;
      // ---- epilogue: dq = scale dQ + the linear part (padding rows 0) ----
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_DONE), u & 1, abort)))) break;
      tc::fence_after_sync();
      // one 32-column chunk at a time; the linear part of the next chunk is loaded while
      // this one is converted
      constexpr int NC = D / 64;  // chunks of this warpgroup's half of the columns
      __nv_bfloat16* dst = prm.dq + ((size_t)bh * prm.N + t) * D;
      const float* acc = (valid && prm.dq_acc) ? prm.dq_acc + ((size_t)bh * prm.N + t) * D : nullptr;
      // NSA's gates: dq += sum_b dlogit_b w_g[h][b]
      float dl[3] = {0.f, 0.f, 0.f};
      const __nv_bfloat16* wg = nullptr;
      if (NSA && prm.dlogit != nullptr && vrow) {
        wg = prm.w_g3 + (size_t)(bh % prm.H) * 3 * D;
#pragma unroll
        for (int x2 = 0; x2 < 3; ++x2) dl[x2] = prm.dlogit[x2 * prm.bstride + (size_t)bh * prm.N + t];
      }
      float4 an[8];
      load_row32(acc, hw * NC, an);
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int ch = hw * NC + c;
        uint32_t v[32];
        if (T > 0) {
          tc::tmem_ld32(tmem + lane_off + 32 * ch, v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        float4 a4[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a4[j] = an[j];
        if (c + 1 < NC) load_row32(acc, ch + 1, an);
        tc::tmem_ld_wait();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4& q4 = a4[j >> 1];
            float a0 = fmaf(prm.scale, __uint_as_float(v[2 * j]), (j & 1) ? q4.z : q4.x);
            float a1 = fmaf(prm.scale, __uint_as_float(v[2 * j + 1]), (j & 1) ? q4.w : q4.y);
            if (NSA && wg != nullptr) {
#pragma unroll
              for (int x2 = 0; x2 < 3; ++x2) {
                const float2 wv = unpack_bf16(*reinterpret_cast<const uint32_t*>(wg + x2 * D + 32 * ch + 2 * j));
                a0 = fmaf(dl[x2], wv.x, a0);
                a1 = fmaf(dl[x2], wv.y, a1);
              }
            }
            w[j] = vrow ? pack_bf16(a0, a1) : 0u;
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
          for (int j = 0; j < 4; ++j) d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(ACC_FREE));
      if (!more) break;
    }
    if (!ok) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <int D, int SL>  // SL ring slots
struct DkvLayout {
  static constexpr int NP = D / 64;
  static constexpr int kOffK = 0;                              // K: 128 keys, NP panels of 16 KB
  static constexpr int kOffV = kOffK + NP * 16384;             // V
  static constexpr int kTile = NP * 8192;                      // one 64-row Q or dO tile
  static constexpr int kSlot = 2 * kTile;                      // Q_i, dO_i
  static constexpr int kOffRing = kOffV + NP * 16384;
  static constexpr int kOffLD = kOffRing + SL * kSlot;         // lse_i, delta_i of each slot (512 bytes)
  static constexpr int kOffBar = kOffLD + SL * 512;
  static constexpr int kOffMisc = kOffBar + 32 * 8;            // TMEM address, abort flag, two unit headers
  static constexpr int kSmem = kOffMisc + 64;
  // TMEM: dV, dK: 2 D; S^T / dP^T: 128; P^T / dS^T: 64 (bf16 pairs); K: D / 2 (the A operand
  // of S^T = K Q_i^T, bf16 pairs)
  static constexpr int kTmemCols = 512;
  static constexpr int kKCol = 2 * D + 192;
  static_assert(kKCol + D / 2 <= kTmemCols, "TMEM columns");
};

struct DkvParams {
  const uint32_t* bits;   // three-way: [B*H][nkb][words] critical; top-n: [B*H_kv][nkb][words] selected
  uint32_t* dlist;        // [units][list_cap]: merged (head, query block) list of each unit
  uint32_t* lbits;        // top-n modes: [units][4][words] the loader's bitmaps of each unit
  const float* lse;       // [B*H][N] (log2 domain); NSA: [3][B*H][N] per branch, gate folded in
  const float* delta;     // [B*H][N]; NSA: [3][B*H][N]
  const float* dk_acc;    // [B*H_kv][N][D] or null
  const float* dv_acc;
  const float* kcol;      // smooth-K: [B*H_kv][D] = -(sum of the linear dk over valid tokens) / N_valid, or null
  __nv_bfloat16* dk;      // [B*H_kv][N][D]
  __nv_bfloat16* dv;
  int* status;
  int* counter;           // units handed out so far (0 at launch)
  int H, group, N, n_valid, nb, npairs, words, window, units;
  float scale, scale_log2;
  int list_cap;           // entries of one unit's list
  int nqb;                // query blocks per head
  size_t bstride;         // NSA: branch stride of lse / delta (B*H*N)
  // NSA tokens: the compressed branch's key gradients dKc (scaled), dVc [B*H_kv][ncmp_pad][D]
  // (fp32, null without compressed keys), scattered back to the tokens of each block
  const float* dkc;
  const float* dvc;
  int n_cmp, ncmp_pad, kstride, kspan;
  float inv_len;          // 1 / cmp_block
  // NSA compressed keys: units are (KV head, pair of compressed tiles, chunk of chunk
  // entries of its (query head, query block) list); items units per KV head; raw dV, dK
  // partials [B*H_kv*items][2][128][D] (fp32)
  float* part;
  int chunk, items;
};

// One dK / dV unit: its KV head, its pair of key blocks and (compressed keys) its chunk.
// Top-n modes take the units pair-major: under the causal mask the early key blocks have
// the longest lists, so the long units of every KV head come first and the short ones
// fill the end (units are handed out one ahead of their start).
struct DkvUnit {
  int bkv, pr, chk;
};
template <bool TOPN, bool NSAC>
__device__ __forceinline__ DkvUnit dkdv_unit(const DkvParams& prm, int x) {
  DkvUnit w{0, 0, 0};
  if (TOPN && !NSAC) {
    const int heads = prm.units / prm.npairs;  // B * H_kv
    w.pr = x / heads;
    w.bkv = x % heads;
  } else if (NSAC) {
    const CmpSplit split{prm.n_cmp, prm.kstride, prm.kspan, prm.nqb, prm.group, prm.chunk};
    w.bkv = x / prm.items;
    int it = x % prm.items, u = 0;
    while (u < split.units() - 1 && it >= split.chunks(u)) it -= split.chunks(u++);
    w.pr = u;
    w.chk = it;
  } else {
    w.bkv = x / prm.npairs;
    w.pr = x % prm.npairs;
  }
  return w;
}

// The merged (query head, query block) list of one dK / dV unit, built by one warp into
// dlist; top-n modes use four bitmaps in `wb` (global scratch of the unit). Returns the
// count (in every lane).
template <bool TOPN, bool NSAT, bool NSAC>
__device__ int dkdv_unit_list(const DkvParams& prm, const DkvUnit& w, uint32_t* dlist, uint32_t* wb, int lane) {
  const int Hkv = prm.H / prm.group;
  const int b = w.bkv / Hkv, hk = w.bkv % Hkv;
  const int j_h[2] = {2 * w.pr, 2 * w.pr + 1};
  const bool valid_j[2] = {j_h[0] < prm.nb, j_h[1] < prm.nb};
  auto head_of = [&](int g) { return b * prm.H + hk * prm.group + g; };
  int n = 0;
  if (NSAC) {
    // chunk ch of the entries (g, i), g-major, i from the first attending block
    const CmpSplit split{prm.n_cmp, prm.kstride, prm.kspan, prm.nqb, prm.group, prm.chunk};
    const int f = split.first_block(w.pr), ni = prm.nqb - f;
    const int e0 = w.chk * prm.chunk, total = split.entries(w.pr);
    const int cnt = total - e0 < prm.chunk ? total - e0 : prm.chunk;
    for (int x = lane; x < cnt; x += 32) {
      const int g = (e0 + x) / ni, i = f + (e0 + x) % ni;
      uint32_t act = 0u;
      for (int h = 0; h < 2; ++h)  // half h is active when block i's last row reaches its first key
        if (valid_j[h] && (long long)j_h[h] * kBlock * prm.kstride + prm.kspan <= (long long)i * kBlock + kBlock - 1)
          act |= 1u << (kActBit + h);
      dlist[x] = (uint32_t)i | act | ((uint32_t)g << kTagShift);
    }
    n = cnt > 0 ? cnt : 0;
  } else if (!TOPN) {
    // every query head of the group: the query blocks that hold j0 or j1 as critical
    for (int g = 0; g < prm.group; ++g) {
      const size_t row = (size_t)head_of(g) * prm.nb;
      n = merge_bitmaps(prm.bits + (row + j_h[0]) * prm.words,
                        prm.bits + (row + (valid_j[1] ? j_h[1] : 0)) * prm.words, nullptr, nullptr, prm.words,
                        valid_j[0], valid_j[1], (uint32_t)g, dlist, n, lane);
    }
  } else {
    // the group shares one selection: the query blocks that selected j0 / j1, plus those
    // whose causal window reaches them (j <= i <= (64 j + 62 + window) / 64); four bitmaps
    // (active 0 / 1, selected 0 / 1)
    for (int h = 0; h < 2; ++h) {
      const uint32_t* selrow = prm.bits + ((size_t)w.bkv * prm.nb + (valid_j[h] ? j_h[h] : 0)) * prm.words;
      int last = j_h[h] - 1;
      if (prm.window > 0) {
        last = (j_h[h] * kBlock + kBlock - 2 + prm.window) / kBlock;
        if (last > prm.nb - 1) last = prm.nb - 1;
      }
      for (int wd = lane; wd < prm.words; wd += 32) {
        const uint32_t sv = valid_j[h] ? selrow[wd] : 0u;
        uint32_t win = 0u;
        if (valid_j[h])
          for (int b2 = 0; b2 < 32; ++b2) {
            const int i = 32 * wd + b2;
            if (i >= j_h[h] && i <= last) win |= 1u << b2;
          }
        wb[h * prm.words + wd] = NSAT ? win : (sv | win);  // NSA: the window branch alone
        wb[(2 + h) * prm.words + wd] = sv;
      }
    }
    __syncwarp();
    for (int g = 0; g < prm.group; ++g) {
      if (NSAT) {  // selected entries (tag 2g), then window entries (tag 2g + 1)
        n = merge_bitmaps(wb + 2 * prm.words, wb + 3 * prm.words, wb + 2 * prm.words, wb + 3 * prm.words, prm.words,
                          valid_j[0], valid_j[1], (uint32_t)(2 * g), dlist, n, lane);
        n = merge_bitmaps(wb, wb + prm.words, nullptr, nullptr, prm.words, valid_j[0], valid_j[1],
                          (uint32_t)(2 * g + 1), dlist, n, lane);
      } else {
        n = merge_bitmaps(wb, wb + prm.words, wb + 2 * prm.words, wb + 3 * prm.words, prm.words, valid_j[0],
                          valid_j[1], (uint32_t)g, dlist, n, lane);
      }
    }
  }
  __syncwarp();
  return n;
}

// TOPN: element (query t, key s) is kept when s <= t and (block(s) selected or s > t - window).
// NSA tokens (kModeNsaTok): selected and window entries are separate (each with its
// branch's log-sum-exp and D), and the epilogue adds the compressed branch's share.
// NSA compressed keys (kModeNsaCmp): tmK / tmV map the compressed keys; key c is kept
// for query t when c < n_cmp and c * kstride + kspan <= t; raw fp32 partials out.
// Persistent: one CTA per SM takes units (pairs of key blocks, or compressed-key items)
// from prm.counter.
template <int D, int MODE, int SL>
__global__ void __launch_bounds__(kBwThreads, 1)
    flash_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      DkvParams prm) {
  constexpr bool TOPN = MODE != kModeThree, NSAT = MODE == kModeNsaTok, NSAC = MODE == kModeNsaCmp;
  using L = DkvLayout<D, SL>;
  constexpr int NP = L::NP, S = SL;
  constexpr uint32_t kAll = 0xffffffffu;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }
  const int Hkv = prm.H / prm.group;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);  // tmem, -, abort, -, headers
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  // header of this CTA's unit u: the unit index (-1: no more units) and its entry count
  auto hdr = [&](int u) { return misc + 4 + 2 * (u & 1); };
  auto unit_list = [&](int x) { return prm.dlist + (size_t)x * prm.list_cap; };
  // list tag -> branch of lse / delta (the query head of the group is tag, or tag / 2 for NSA tokens)
  auto tag_branch = [&](uint32_t tag) { return NSAT ? (int)kBrSel + (int)(tag & 1u) : NSAC ? (int)kBrCmp : 0; };
  // ring slots: LOADED (Q_i, dO_i, lse_i, delta_i landed), SLOT_FREE (the dV / dK products
  // read them); one S^T / dP^T buffer: SP_FULL (products done), S_READ (row warps have
  // loaded them); one P^T / dS^T buffer: DS_FULL (written), PS_FREE (dV / dK products
  // done). Per unit: LIST_FULL / LIST_FREE (its header, two buffers), K_FULL / V_FULL (K, V
  // landed), K_TMEM (row warps have copied K into TMEM), PROD_DONE (its S^T / dP^T products
  // are done: V and the K columns may be overwritten), ACC_DONE (dV, dK complete), ACC_FREE
  // (row warps have read them)
  constexpr int LOADED = 0, SLOT_FREE = S, SP_FULL = 2 * S, S_READ = SP_FULL + 1, DS_FULL = S_READ + 1,
                PS_FREE = DS_FULL + 1, LIST_FULL = PS_FREE + 1, LIST_FREE = LIST_FULL + 2, K_FULL = LIST_FREE + 2,
                V_FULL = K_FULL + 1, K_TMEM = V_FULL + 1, PROD_DONE = K_TMEM + 1, ACC_DONE = PROD_DONE + 1,
                ACC_FREE = ACC_DONE + 1, CLAIM = ACC_FREE + 1;
  static_assert(CLAIM < 32, "mbarriers");
  const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sR = sbase + L::kOffRing;

  if (tid == 0) {
    misc[2] = 0;
    for (int x = 0; x < S; ++x) {
      tc::mbar_init(bar(LOADED + x), 1);
      tc::mbar_init(bar(SLOT_FREE + x), 1);
    }
    tc::mbar_init(bar(SP_FULL), 1);
    tc::mbar_init(bar(S_READ), kRowWarps);
    tc::mbar_init(bar(DS_FULL), kRowWarps);
    tc::mbar_init(bar(PS_FREE), 1);
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar(LIST_FULL + x), 1);
      tc::mbar_init(bar(LIST_FREE + x), kListReaders);
    }
    tc::mbar_init(bar(K_FULL), 1);
    tc::mbar_init(bar(V_FULL), 1);
    tc::mbar_init(bar(K_TMEM), kRowWarps);
    tc::mbar_init(bar(PROD_DONE), 1);
    tc::mbar_init(bar(ACC_DONE), 1);
    tc::mbar_init(bar(ACC_FREE), kRowWarps);
    tc::mbar_init(bar(CLAIM), 1);
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(sbase + L::kOffMisc, L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 2;
  bool ok = true;

  if (warp == kLoadWarp) {
    // ======================= unit loader ======================================
    // the next unit's list, then its K (once the row warps have copied the previous K into
    // TMEM) and V (once the previous unit's products are done)
    int prev = -1;
    for (int u = 0;; ++u) {
      // the next unit is taken once the producer is within kClaimLead tiles of the current
      // unit's end: a unit is committed to this CTA only shortly before it can start
      if (u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(CLAIM), (u - 1) & 1, abort));
      if (!ok) break;
      int x = 0;
      if (lane == 0) x = atomicAdd(prm.counter, 1);
      x = __shfl_sync(kAll, x, 0);
      if (u >= 2) ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FREE + (u & 1)), ((u - 2) >> 1) & 1, abort));
      if (!ok) break;
      volatile int* h = hdr(u);
      if (x >= prm.units) {
        if (lane == 0) {
          h[0] = -1;
          h[1] = 0;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(LIST_FULL + (u & 1)));
        break;
      }
      const DkvUnit w = dkdv_unit<TOPN, NSAC>(prm, x);
      uint32_t* wb = prm.lbits ? prm.lbits + (size_t)x * 4 * prm.words : nullptr;
      const int n = dkdv_unit_list<TOPN, NSAT, NSAC>(prm, w, unit_list(x), wb, lane);
      if (lane == 0) {
        h[0] = x;
        h[1] = n;
      }
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(bar(LIST_FULL + (u & 1)));
        if (u >= 1) ok = tc::mbar_wait(bar(K_TMEM), (u - 1) & 1, abort);
        if (ok) {
          tc::mbar_expect_tx(bar(K_FULL), 2 * NP * 8192);
          for (int hf = 0; hf < 2; ++hf)
            for (int p = 0; p < NP; ++p)
              tc::tma_load_3d(sK + p * 16384 + hf * 8192, &tmK, bar(K_FULL), 64 * p, (2 * w.pr + hf) * kBlock, w.bkv);
        }
        if (ok && u >= 1) ok = tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort);
        if (ok) {
          tc::mbar_expect_tx(bar(V_FULL), 2 * NP * 8192);
          for (int hf = 0; hf < 2; ++hf)
            for (int p = 0; p < NP; ++p)
              tc::tma_load_3d(sV + p * 16384 + hf * 8192, &tmV, bar(V_FULL), 64 * p, (2 * w.pr + hf) * kBlock, w.bkv);
          // the previous unit's epilogue reads its linear parts next: into L2 ahead of it
          if (prev >= 0 && prm.dk_acc != nullptr) {
            const int t0 = 2 * (prev % prm.npairs) * kBlock;
            const int rows = prm.N - t0 < 2 * kBlock ? prm.N - t0 : 2 * kBlock;
            const size_t off = ((size_t)(prev / prm.npairs) * prm.N + t0) * D;
            tc::prefetch_l2(prm.dv_acc + off, (uint32_t)rows * D * 4);
            tc::prefetch_l2(prm.dk_acc + off, (uint32_t)rows * D * 4);
          }
        }
      }
      ok = __shfl_sync(kAll, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      prev = x;
    }
    if (ok && lane == 0 && prev >= 0 && prm.dk_acc != nullptr) {  // the last unit's linear parts
      const int t0 = 2 * (prev % prm.npairs) * kBlock;
      const int rows = prm.N - t0 < 2 * kBlock ? prm.N - t0 : 2 * kBlock;
      const size_t off = ((size_t)(prev / prm.npairs) * prm.N + t0) * D;
      tc::prefetch_l2(prm.dv_acc + off, (uint32_t)rows * D * 4);
      tc::prefetch_l2(prm.dk_acc + off, (uint32_t)rows * D * 4);
    }
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp == kProdWarp) {
    // ======================= TMA producer: the Q / dO ring, across units =======
    if (lane == 0) {
      int g = 0;  // tiles of this CTA so far
      for (int u = 0;; ++u) {
        if (!(ok = tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort))) break;
        const int x = hdr(u)[0], T = hdr(u)[1];
        if (x < 0) break;
        const uint32_t* dl = unit_list(x);
        const int bkv = dkdv_unit<TOPN, NSAC>(prm, x).bkv;
        const int bh0 = (bkv / Hkv) * prm.H + (bkv % Hkv) * prm.group;  // the group's first query head
        uint32_t e_next = T > 0 ? dl[0] : 0u;  // list entries are read one tile ahead
        const int claim_at = T > kClaimLead ? T - kClaimLead : 0;
        if (claim_at == 0) tc::mbar_arrive(bar(CLAIM));
        for (int m = 0; m < T && ok; ++m, ++g) {
          if (m == claim_at && m > 0) tc::mbar_arrive(bar(CLAIM));
          const int slot = g % S;
          const uint32_t e = e_next;
          if (m + 1 < T) e_next = dl[m + 1];
          if (g >= S && !(ok = tc::mbar_wait(bar(SLOT_FREE + slot), ((g / S) - 1) & 1, abort))) break;
          const int i = (int)(e & kIdxMask), bh = bh0 + (int)(NSAT ? (e >> kTagShift) >> 1 : e >> kTagShift);
          const size_t boff = (size_t)tag_branch(e >> kTagShift) * prm.bstride;
          const uint32_t dst = sR + slot * L::kSlot;
          tc::mbar_expect_tx(bar(LOADED + slot), 2 * L::kTile + 512);
          for (int p = 0; p < NP; ++p) {
            tc::tma_load_3d(dst + p * 8192, &tmQ, bar(LOADED + slot), 64 * p, i * kBlock, bh);
            tc::tma_load_3d(dst + L::kTile + p * 8192, &tmO, bar(LOADED + slot), 64 * p, i * kBlock, bh);
          }
          const uint32_t ld = sbase + L::kOffLD + slot * 512;
          tc::bulk_load(ld, prm.lse + boff + (size_t)bh * prm.N + i * kBlock, 256, bar(LOADED + slot));
          tc::bulk_load(ld + 256, prm.delta + boff + (size_t)bh * prm.N + i * kBlock, 256, bar(LOADED + slot));
        }
        tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      }
      // the last release of every slot: no product reads the ring and no commit is in flight at exit
      for (int m = (g > S ? g - S : 0); m < g && ok; ++m)
        ok = tc::mbar_wait(bar(SLOT_FREE + m % S), (m / S) & 1, abort);
      if (!ok) {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= S^T / dP^T issuer ================================
    constexpr uint32_t kIdS = tc::idesc_bf16(128, 64, false, false);
    // base descriptors; a byte offset off is added as off >> 4 (start-address field)
    const uint64_t dVd = tc::sw128_desc(sV, 16, 1024);
    const uint64_t dRk = tc::sw128_desc(sR, 16, 1024);    // ring tiles, K-major
    // S^T = K Q_i^T (A = K in TMEM: only Q_i is read from shared memory, full rate at
    // N = 64), dP^T = V dO_i^T (M = 128 keys, N = 64 queries) into the S buffer
    auto issue_sp = [&](int g) {
      const uint32_t so = (uint32_t)((g % S) * L::kSlot);
      const uint32_t tS = tmem + 2 * D;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ko = (uint32_t)((k >> 2) * 16384 + (k & 3) * 32), qo = (uint32_t)((k >> 2) * 8192 + (k & 3) * 32);
        tc::mma_bf16_ts(tS, tmem + L::kKCol + 8 * k, dRk + ((so + qo) >> 4), kIdS, k > 0);
        tc::mma_bf16_ss(tS + 64, dVd + (ko >> 4), dRk + ((so + L::kTile + qo) >> 4), kIdS, k > 0);
      }
      tc::mma_commit(bar(SP_FULL));
    };
    int g = 0, u = 0;
    for (;; ++u) {
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort)))) break;
      const int x = hdr(u)[0], T = hdr(u)[1];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (x < 0) break;
      ok = __all_sync(kAll, tc::mbar_wait(bar(K_TMEM), u & 1, abort)) &&
           __all_sync(kAll, tc::mbar_wait(bar(V_FULL), u & 1, abort));
      if (!ok) break;
      tc::fence_after_sync();
      for (int m = 0; m < T && ok; ++m, ++g) {
        // the S buffer is free once the row warps have loaded S^T_{g-1}, dP^T_{g-1}: the
        // products of tile g run while they compute P^T_{g-1} and dS^T_{g-1}
        if (g >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(S_READ), (g - 1) & 1, abort));
        ok = ok && __all_sync(kAll, tc::mbar_wait(bar(LOADED + g % S), (g / S) & 1, abort));
        tc::fence_after_sync();
        if (ok && tc::elect_one()) {
          issue_sp(g);
          if (m == T - 1) tc::mma_commit(bar(PROD_DONE));
        }
        __syncwarp();
      }
      if (ok && T == 0 && tc::elect_one()) tc::mma_commit(bar(PROD_DONE));
      __syncwarp();
      if (!ok) break;
    }
    // the last unit's PROD_DONE has landed before the CTA exits
    if (ok && u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort));
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp == kDqWarp) {
    // ======================= dV / dK issuer ===================================
    constexpr uint32_t kIdA = tc::idesc_bf16(128, D, false, true);
    const uint64_t dRn = tc::sw128_desc(sR, 8192, 1024);  // ring tiles, N-major (64-row panels)
    int g = 0, u = 0;
    for (;; ++u) {
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + (u & 1)), (u >> 1) & 1, abort)))) break;
      const int x = hdr(u)[0], T = hdr(u)[1];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (x < 0) break;
      // the accumulators are free once the row warps have read the previous unit's
      if (u >= 1 && !(ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_FREE), (u - 1) & 1, abort)))) break;
      for (int m = 0; m < T && ok; ++m, ++g) {
        if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(DS_FULL), g & 1, abort)))) break;
        tc::fence_after_sync();
        if (tc::elect_one()) {
          // dV += P^T dO_i, dK += dS^T Q_i: A = P^T / dS^T from their TMEM buffer (bf16 pairs),
          // B = dO_i / Q_i N-major. The slot is released after these products: S^T_g, dP^T_g
          // (its other readers) completed before the row warps could write P^T_g, dS^T_g
          const uint32_t so = (uint32_t)((g % S) * L::kSlot);
          const uint32_t tP = tmem + 2 * D + 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (m > 0 || kk > 0) ? 1u : 0u;
            tc::mma_bf16_ts(tmem, tP + 8 * kk, dRn + ((so + L::kTile + kk * 2048) >> 4), kIdA, acc);
            tc::mma_bf16_ts(tmem + D, tP + 32 + 8 * kk, dRn + ((so + kk * 2048) >> 4), kIdA, acc);
          }
          tc::mma_commit(bar(SLOT_FREE + g % S));
          tc::mma_commit(bar(PS_FREE));
          if (m == T - 1) tc::mma_commit(bar(ACC_DONE));
        }
        __syncwarp();
      }
      if (ok && T == 0 && tc::elect_one()) tc::mma_commit(bar(ACC_DONE));
      __syncwarp();
      if (!ok) break;
    }
    // the last release of the P / dS buffer and the last ACC_DONE: no commit is in flight at exit
    if (ok && g > 0) ok = __all_sync(kAll, tc::mbar_wait(bar(PS_FREE), (g - 1) & 1, abort));
    if (ok && u >= 1) ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_DONE), (u - 1) & 1, abort));
    if (!ok && lane == 0) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  } else if (warp < kRowWarps) {
    // ======================= rows (keys): P^T and dS^T, then the epilogue =====
    // warp = quarter (TMEM lanes) + 4 * hw (query columns 32 hw .. 32 hw + 31 of each tile)
    const int quarter = warp & 3, hw = warp >> 2;
    const int r = quarter * 32 + lane, hf = r >> 6;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = prm.scale_log2;
    // key row r (the TMEM lane) into columns kKCol.. as bf16 pairs, this warpgroup's half of
    // the features, from the swizzled K tile (16-byte chunk c of a row at c ^ (row & 7)),
    // once unit u's K has landed and the previous unit's S^T products are done
    auto copy_k = [&](int u) {
      bool fine = true;
      if (u >= 1) fine = __all_sync(kAll, tc::mbar_wait(bar(PROD_DONE), (u - 1) & 1, abort));
      fine = fine && __all_sync(kAll, tc::mbar_wait(bar(K_FULL), u & 1, abort));
      if (fine) {
        tc::fence_after_sync();
        constexpr int CH = D / 16;  // 16-byte chunks per warpgroup half: 8 (D = 128) or 4
        uint32_t kv[CH * 4];
#pragma unroll
        for (int x2 = 0; x2 < CH; ++x2) {
          const int chunk = hw * CH + x2;  // of the row's D / 8 chunks
          const int p = chunk >> 3, c = chunk & 7;
          const uint4 v4 = *reinterpret_cast<const uint4*>(smem + L::kOffK + p * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
          kv[4 * x2] = v4.x; kv[4 * x2 + 1] = v4.y; kv[4 * x2 + 2] = v4.z; kv[4 * x2 + 3] = v4.w;
        }
        if constexpr (CH * 4 == 32)
          tc::tmem_st32(tmem + lane_off + L::kKCol + 32 * hw, *reinterpret_cast<const uint32_t(*)[32]>(kv));
        else
          tc::tmem_st16(tmem + lane_off + L::kKCol + 16 * hw, *reinterpret_cast<const uint32_t(*)[16]>(kv));
        tc::tmem_st_wait();
      }
      tc::fence_async_smem();  // the K tile's reads come before the next unit's load into it
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(K_TMEM));
      return fine;
    };
    int g = 0;
    ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL), 0, abort));
    if (ok && hdr(0)[0] >= 0) ok = copy_k(0);
    for (int u = 0; ok; ++u) {
      const int x = hdr(u)[0], T = hdr(u)[1];
      if (x < 0) break;
      const uint32_t* dl = unit_list(x);
      const DkvUnit w = dkdv_unit<TOPN, NSAC>(prm, x);
      const int j_h = 2 * w.pr + hf;  // this row's key block
      const bool valid_j = j_h < prm.nb;
      const int key = j_h * kBlock + (r & 63);  // NSA compressed keys: the compressed key index
      const bool vkey = valid_j && key < (NSAC ? prm.n_cmp : prm.n_valid);
      const int k_w = j_h * kBlock + ((quarter * 32) & 63);  // first key of this warp
      uint32_t e_next = T > 0 ? dl[0] : 0u;  // list entries are read one tile ahead
      for (int m = 0; m < T && ok; ++m, ++g) {
        const int slot = g % S;
        const uint32_t e = e_next;
        if (m + 1 < T) e_next = dl[m + 1];
        const bool act = vkey && ((e >> (kActBit + hf)) & 1u);
        const bool sel = (e >> (kSelBit + hf)) & 1u;
        const int t0 = (int)(e & kIdxMask) * kBlock + 32 * hw;  // first query token of this half
        ok = __all_sync(kAll, tc::mbar_wait(bar(SP_FULL), g & 1, abort)) &&
             __all_sync(kAll, tc::mbar_wait(bar(LOADED + slot), (g / S) & 1, abort));
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t tS = tmem + lane_off + 2 * D;
        uint32_t sv[32], pv[32];
        tc::tmem_ld32(tS + 32 * hw, sv);
        tc::tmem_ld32(tS + 64 + 32 * hw, pv);
        // this half's log-sum-exp and D values (one per query column), read as pairs below
        const uint64_t* lse2 = reinterpret_cast<const uint64_t*>(smem + L::kOffLD + slot * 512) + 16 * hw;
        const uint64_t* dl2 = lse2 + 32;
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(S_READ));
        // warp-uniform: every (key, query) of this warp's 32 x 32 sub-tile is kept (keys
        // k_w .. k_w + 31 all valid), so no per-element mask
        const bool act_w = valid_j && ((e >> (kActBit + hf)) & 1u);
        bool full = act_w && k_w + 31 < (NSAC ? prm.n_cmp : prm.n_valid);
        if (NSAC)
          full = full && (k_w + 31) * prm.kstride + prm.kspan <= t0;
        else if (TOPN)
          full = full && k_w + 31 <= t0 && (sel || k_w > t0 + 31 - prm.window);
        // P^T = 2^(s * scale * log2 e - lse), dS^T = P^T (dP^T - D), two columns per packed op
        const uint64_t sc2 = tc::f2_pack(sl2, sl2);
        uint32_t pw[16], dw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) pw[j] = dw[j] = 0u;  // a half that does not use the tile
        if (act_w)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint64_t y = tc::fsub2(tc::fmul2(tc::f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), sc2),
                                       lse2[j]);
          float p0 = tc::ex2_approx(tc::f2_lo(y)), p1 = tc::ex2_approx(tc::f2_hi(y));
          if (!full) {
            bool keep[2];
#pragma unroll
            for (int x2 = 0; x2 < 2; ++x2) {
              const int c = 2 * j + x2;
              keep[x2] = act;
              if (NSAC)
                keep[x2] = keep[x2] && key * prm.kstride + prm.kspan <= t0 + c;
              else if (TOPN)
                keep[x2] = keep[x2] && key <= t0 + c && (sel || key > t0 + c - prm.window);
            }
            p0 = keep[0] ? p0 : 0.f;
            p1 = keep[1] ? p1 : 0.f;
          }
          const uint64_t p2 = tc::f2_pack(p0, p1);
          const uint64_t d2 = tc::fmul2(p2, tc::fsub2(tc::f2_pack(__uint_as_float(pv[2 * j]), __uint_as_float(pv[2 * j + 1])),
                                                      dl2[j]));
          pw[j] = pack_bf16(p0, p1);
          dw[j] = pack_bf16(tc::f2_lo(d2), tc::f2_hi(d2));
        }
        // the P / dS buffer was last read by the products of tile g - 1 (PS_FREE has then
        // completed g - 1 or g phases: the products of tile g need this tile's P and dS)
        if (g >= 1 && !(ok = __all_sync(kAll, tc::mbar_wait(bar(PS_FREE), (g - 1) & 1, abort)))) break;
        tc::fence_after_sync();
        const uint32_t tP = tmem + lane_off + 2 * D + 128;
        tc::tmem_st16(tP + 16 * hw, pw);
        tc::tmem_st16(tP + 32 + 16 * hw, dw);
        tc::tmem_st_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(DS_FULL));
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(LIST_FREE + (u & 1)));
      if (!ok) break;
      // the next unit's K into TMEM before this unit's epilogue, so that its first products
      // run meanwhile
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(LIST_FULL + ((u + 1) & 1)), ((u + 1) >> 1) & 1, abort)))) break;
      const bool more = hdr(u + 1)[0] >= 0;
      if (more && !(ok = copy_k(u + 1))) break;
      // ---- epilogue ----
      if (!(ok = __all_sync(kAll, tc::mbar_wait(bar(ACC_DONE), u & 1, abort)))) break;
      tc::fence_after_sync();
      if (NSAC) {
        // raw partial sums of this chunk (every row, zero where nothing was accumulated)
        float* prt = prm.part + (size_t)x * 2 * 128 * D;
        for (int which = 0; which < 2; ++which) {
          float* dst = prt + ((size_t)which * 128 + r) * D;
#pragma unroll 1
          for (int c2 = hw * (D / 64); c2 < (hw + 1) * (D / 64); ++c2) {
            uint32_t v[32];
            if (T > 0) {
              tc::tmem_ld32(tmem + lane_off + which * D + 32 * c2, v);
              tc::tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0u;
            }
            float4* d4 = reinterpret_cast<float4*>(dst + 32 * c2);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]), __uint_as_float(v[4 * j + 2]),
                                  __uint_as_float(v[4 * j + 3]));
          }
        }
      } else {
        // dk = scale dK + linear part, dv = dV + linear part (padding keys 0), one 32-column
        // chunk at a time (dV's, then dK's); the linear part of the next chunk is loaded
        // while this one is converted
        const size_t row = (size_t)w.bkv * prm.N + key;
        // NSA: the compressed blocks c that hold token `key` (c * kstride <= key <= c * kstride + kspan)
        int c_lo = 0, c_hi = -1;
        if (NSAT && prm.dkc != nullptr && vkey) {
          c_lo = key <= prm.kspan ? 0 : (key - prm.kspan + prm.kstride - 1) / prm.kstride;
          c_hi = key / prm.kstride;
          if (c_hi > prm.n_cmp - 1) c_hi = prm.n_cmp - 1;
        }
        constexpr int NC = D / 64;  // chunks of this warpgroup's half of the columns
        const float* accv = (valid_j && prm.dv_acc) ? prm.dv_acc + row * D : nullptr;
        const float* acck = (valid_j && prm.dk_acc) ? prm.dk_acc + row * D : nullptr;
        float4 an[8];
        load_row32(accv, hw * NC, an);
#pragma unroll
        for (int idx = 0; idx < 2 * NC; ++idx) {
          const int which = idx / NC, ch = hw * NC + idx % NC;
          uint32_t v[32];
          if (T > 0) {
            tc::tmem_ld32(tmem + lane_off + which * D + 32 * ch, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0u;
          }
          float4 a4[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) a4[j] = an[j];
          if (idx + 1 < 2 * NC) {
            const int wn = (idx + 1) / NC, chn = hw * NC + (idx + 1) % NC;
            load_row32(wn == 0 ? accv : acck, chn, an);
          }
          tc::tmem_ld_wait();
          if (!valid_j) continue;  // keys past the last block: nothing to write
          __nv_bfloat16* dst = (which == 0 ? prm.dv : prm.dk) + row * D;
          const float* kc = (which == 1 && prm.kcol) ? prm.kcol + (size_t)w.bkv * D : nullptr;
          const float sc = which == 0 ? 1.f : prm.scale;
          uint32_t wv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4& q4 = a4[j >> 1];
            float a0 = fmaf(sc, __uint_as_float(v[2 * j]), (j & 1) ? q4.z : q4.x);
            float a1 = fmaf(sc, __uint_as_float(v[2 * j + 1]), (j & 1) ? q4.w : q4.y);
            if (kc) {  // smooth-K: the mean key's share of the gradient
              a0 += kc[32 * ch + 2 * j];
              a1 += kc[32 * ch + 2 * j + 1];
            }
            if (NSAT) {  // compressed keys and values are block means: each token gets 1 / length
              const float* cg = which == 0 ? prm.dvc : prm.dkc;
              for (int cc = c_lo; cc <= c_hi; ++cc) {
                const float2 xx = *reinterpret_cast<const float2*>(cg + ((size_t)w.bkv * prm.ncmp_pad + cc) * D + 32 * ch + 2 * j);
                a0 = fmaf(prm.inv_len, xx.x, a0);
                a1 = fmaf(prm.inv_len, xx.y, a1);
              }
            }
            wv[j] = vkey ? pack_bf16(a0, a1) : 0u;
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
          for (int j = 0; j < 4; ++j) d4[j] = make_uint4(wv[4 * j], wv[4 * j + 1], wv[4 * j + 2], wv[4 * j + 3]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(ACC_FREE));
      if (!more) break;
    }
    if (!ok) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// capacity of the dQ kernel's merged block list (at least 1)
static int dq_list_cap(const Plan& p) {
  const sla_config& c = p.c;
  const bool topn = c.mode == SLA_MODE_TOPN_WINDOW;
  int per_half = topn ? c.top_n : c.k_h;
  if (topn) per_half += (c.window + 62) / kBlock + 2;  // selected blocks plus the window's reach
  int cap = 2 * per_half < p.nkb ? 2 * per_half : p.nkb;
  if (topn && c.nsa_branches) {  // compressed tiles, then the selected and the window blocks (two halves each)
    const int sel = 2 * c.top_n < p.nkb ? 2 * c.top_n : p.nkb;
    const int win = 2 * ((c.window + 62) / kBlock + 2) < p.nkb ? 2 * ((c.window + 62) / kBlock + 2) : p.nkb;
    cap = p.ncmp_pad / kBlock + sel + win;
  }
  return cap > 0 ? cap : 1;
}

static bool map64(CUtensorMap* m, const void* base, int heads, int n_rows, int N, int D) {
  return make_tmap_3d(m, base, (uint64_t)D, (uint64_t)n_rows, (uint64_t)heads, (uint64_t)D * 2,
                      (uint64_t)N * D * 2, 64, 64);
}

template <int D, int MODE, int SL>
static cudaError_t launch_dq_slots(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);

// shared memory of the dQ kernel: tiles, ring, barriers, two unit lists, the loader's bitmaps
template <int D, int SL>
static int dq_smem(const Plan& p) {
  return DqLayout<D, SL>::kOffList + 2 * dq_list_cap(p) * 4 + 4 * ((p.nkb + 31) / 32) * 4;
}

// the persistent kernels' grid: one CTA per SM (each holds all 512 TMEM columns), at most
// one per unit; the unit counter is zeroed on the stream first
static cudaError_t persistent_grid(int units, int* counter, cudaStream_t s, unsigned* grid) {
  int dev = 0, sms = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(counter, 0, sizeof(int), s)) != cudaSuccess) return e;
  *grid = (unsigned)(units < sms ? units : sms);
  return cudaSuccess;
}

// five ring slots where they fit in shared memory (the K / V loads then start one tile
// earlier), else four
template <int D, int MODE>
static cudaError_t launch_dq_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  return dq_smem<D, 5>(p) <= 227 * 1024 ? launch_dq_slots<D, MODE, 5>(p, bp, a, s)
                                       : launch_dq_slots<D, MODE, 4>(p, bp, a, s);
}

template <int D, int MODE, int SL>
static cudaError_t launch_dq_slots(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  using L = DqLayout<D, SL>;
  constexpr bool TOPN = MODE != kModeThree, NSA = MODE == kModeNsa;
  const sla_config& c = p.c;
  CUtensorMap mq, mo, mk, mv, mkc, mvc;
  if (!map64(&mq, a.q, c.B * c.H, c.N_valid, c.N, D) || !map64(&mo, a.dout, c.B * c.H, c.N_valid, c.N, D) ||
      !map64(&mk, a.k, c.B * c.H_kv, c.N_valid, c.N, D) || !map64(&mv, a.v, c.B * c.H_kv, c.N_valid, c.N, D))
    return cudaErrorInvalidValue;
  // NSA's compressed keys and values (rows beyond n_cmp read as zero); otherwise unused
  const int crows = NSA && p.n_cmp > 0 ? p.n_cmp : 1;
  if (!map64(&mkc, NSA ? (const void*)(a.ws + p.off_kc) : (const void*)a.k, c.B * c.H_kv, crows,
             NSA ? p.ncmp_pad : c.N, D) ||
      !map64(&mvc, NSA ? (const void*)(a.ws + p.off_vc) : (const void*)a.v, c.B * c.H_kv, crows,
             NSA ? p.ncmp_pad : c.N, D))
    return cudaErrorInvalidValue;
  DqParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.crit = reinterpret_cast<const int32_t*>(a.ws + p.off_crit);
  prm.lse = NSA ? reinterpret_cast<const float*>(a.bws + bp.off_lse3) : reinterpret_cast<const float*>(a.ws + p.off_lse);
  prm.delta = reinterpret_cast<const float*>(a.bws + bp.off_delta);
  prm.dq_acc = bp.lin ? reinterpret_cast<const float*>(a.bws + bp.off_dqacc) : nullptr;
  prm.dq = a.dq;
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = p.nkb;
  prm.len = TOPN ? c.top_n : c.k_h;
  prm.npairs = (p.nqb + 1) / 2;
  prm.words = (p.nkb + 31) / 32;
  prm.window = c.window;
  prm.scale = p.scale;
  prm.scale_log2 = p.scale * 1.4426950408889634f;
  prm.bstride = (size_t)c.B * c.H * c.N;
  if (NSA) {
    prm.dlogit = c.has_gate ? reinterpret_cast<const float*>(a.bws + bp.off_dlogit) : nullptr;
    prm.w_g3 = c.has_gate ? a.w_g : nullptr;
    prm.n_cmp = p.n_cmp;
    prm.nct = p.ncmp_pad / kBlock;
    prm.kstride = c.cmp_stride;
    prm.kspan = c.cmp_block - 1;
  }
  prm.units = c.B * c.H * prm.npairs;
  prm.list_cap = dq_list_cap(p);
  prm.counter = reinterpret_cast<int*>(a.bws + bp.off_ctr);
  int smem = dq_smem<D, SL>(p);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM: it holds all 512 TMEM columns
  cudaError_t e = cudaFuncSetAttribute(flash_dq_kernel<D, MODE, SL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = persistent_grid(prm.units, prm.counter, s, &grid)) != cudaSuccess) return e;
  if (grid == 0) return cudaSuccess;
  flash_dq_kernel<D, MODE, SL><<<grid, kBwThreads, smem, s>>>(mq, mo, mk, mv, mkc, mvc, prm);
  return cudaGetLastError();
}

cudaError_t launch_flash_dq(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const int mode = p.c.mode == SLA_MODE_THREEWAY ? kModeThree : p.c.nsa_branches ? kModeNsa : kModeTopn;
  if (p.c.d == 128) {
    if (mode == kModeNsa) return launch_dq_t<128, kModeNsa>(p, bp, a, s);
    return mode == kModeTopn ? launch_dq_t<128, kModeTopn>(p, bp, a, s) : launch_dq_t<128, kModeThree>(p, bp, a, s);
  }
  if (mode == kModeNsa) return launch_dq_t<64, kModeNsa>(p, bp, a, s);
  return mode == kModeTopn ? launch_dq_t<64, kModeTopn>(p, bp, a, s) : launch_dq_t<64, kModeThree>(p, bp, a, s);
}

// entries of one (KV head, pair of key blocks) unit's list in the dK / dV kernel
int dkdv_list_cap(const Plan& p) { return p.group * p.nqb * (p.c.nsa_branches ? 2 : 1); }

// NSA's compressed keys: entries per item, chosen so that the items fill the GPU about
// four times over (at least 64 entries, so that an item's fixed cost stays small)
CmpSplit cmp_split(const Plan& p) {
  const sla_config& c = p.c;
  CmpSplit sp{p.n_cmp, c.cmp_stride, c.cmp_block - 1, p.nqb, p.group, 1 << 30};
  long long total = 0;
  for (int u = 0; u < sp.units(); ++u) total += sp.entries(u);
  total *= (long long)c.B * c.H_kv;
  long long ch = (total + 148 * 4 - 1) / (148 * 4);
  if (ch < 64) ch = 64;
  if (ch > (1 << 20)) ch = 1 << 20;
  sp.chunk = (int)ch;
  return sp;
}

template <int D, int MODE, int SL>
static cudaError_t launch_dkdv_slots(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s);

// shared memory of the dK / dV kernel: tiles, ring, lse / delta, barriers
template <int D, int MODE, int SL>
static int dkdv_smem(const Plan&) {
  return DkvLayout<D, SL>::kSmem;
}

// five ring slots where they fit in shared memory, else four
template <int D, int MODE>
static cudaError_t launch_dkdv_t(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  return dkdv_smem<D, MODE, 5>(p) <= 227 * 1024 ? launch_dkdv_slots<D, MODE, 5>(p, bp, a, s)
                                               : launch_dkdv_slots<D, MODE, 4>(p, bp, a, s);
}

template <int D, int MODE, int SL>
static cudaError_t launch_dkdv_slots(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  constexpr bool NSAT = MODE == kModeNsaTok, NSAC = MODE == kModeNsaCmp;
  const sla_config& c = p.c;
  CUtensorMap mq, mo, mk, mv;
  // NSA's compressed keys: the key tiles are the compressed keys and values
  const void* kb = NSAC ? (const void*)(a.ws + p.off_kc) : (const void*)a.k;
  const void* vb = NSAC ? (const void*)(a.ws + p.off_vc) : (const void*)a.v;
  const int krows = NSAC ? (p.n_cmp > 0 ? p.n_cmp : 1) : c.N_valid, kstride_rows = NSAC ? p.ncmp_pad : c.N;
  if (!map64(&mq, a.q, c.B * c.H, c.N_valid, c.N, D) || !map64(&mo, a.dout, c.B * c.H, c.N_valid, c.N, D) ||
      !map64(&mk, kb, c.B * c.H_kv, krows, kstride_rows, D) || !map64(&mv, vb, c.B * c.H_kv, krows, kstride_rows, D))
    return cudaErrorInvalidValue;
  DkvParams prm;
  memset(&prm, 0, sizeof(prm));
  const bool nsa = NSAT || NSAC;
  prm.bits = reinterpret_cast<const uint32_t*>(a.bws + bp.off_bits);
  prm.dlist = reinterpret_cast<uint32_t*>(a.bws + (NSAC ? bp.off_clist : bp.off_dlist));
  prm.lbits = bp.off_lbits && MODE != kModeThree && !NSAC ? reinterpret_cast<uint32_t*>(a.bws + bp.off_lbits) : nullptr;
  if (MODE != kModeThree && !NSAC && prm.lbits == nullptr) return cudaErrorInvalidValue;
  prm.lse = nsa ? reinterpret_cast<const float*>(a.bws + bp.off_lse3) : reinterpret_cast<const float*>(a.ws + p.off_lse);
  prm.delta = reinterpret_cast<const float*>(a.bws + bp.off_delta);
  prm.dk_acc = bp.lin ? reinterpret_cast<const float*>(a.bws + bp.off_dkacc) : nullptr;
  prm.dv_acc = bp.lin ? reinterpret_cast<const float*>(a.bws + bp.off_dvacc) : nullptr;
  prm.kcol = bp.lin && c.smooth_k ? reinterpret_cast<const float*>(a.bws + bp.off_kcol) : nullptr;
  prm.dk = a.dk;
  prm.dv = a.dv;
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = NSAC ? p.ncmp_pad / kBlock : p.nkb;
  prm.npairs = (prm.nb + 1) / 2;
  prm.words = bp.words;
  prm.window = c.window;
  prm.scale = p.scale;
  prm.scale_log2 = p.scale * 1.4426950408889634f;
  prm.nqb = p.nqb;
  prm.bstride = (size_t)c.B * c.H * c.N;
  prm.list_cap = dkdv_list_cap(p);
  if (nsa) {
    prm.n_cmp = p.n_cmp;
    prm.ncmp_pad = p.ncmp_pad;
    prm.kstride = c.cmp_stride;
    prm.kspan = c.cmp_block - 1;
    prm.inv_len = 1.f / (float)c.cmp_block;
    if (NSAT && p.n_cmp > 0) {
      prm.dkc = reinterpret_cast<const float*>(a.bws + bp.off_dkc);
      prm.dvc = reinterpret_cast<const float*>(a.bws + bp.off_dvc);
    }
  }
  unsigned grid = (unsigned)(c.B * c.H_kv * prm.npairs);
  if (NSAC) {
    const CmpSplit sp = cmp_split(p);
    prm.chunk = sp.chunk;
    prm.items = bp.cmp_items;
    prm.list_cap = sp.chunk;
    prm.part = reinterpret_cast<float*>(a.bws + bp.off_part);
    grid = (unsigned)(c.B * c.H_kv * bp.cmp_items);
    if (grid == 0) return cudaSuccess;
  }
  prm.units = (int)grid;
  prm.counter = reinterpret_cast<int*>(a.bws + bp.off_ctr) + (NSAC ? 2 : 1);
  int smem = dkdv_smem<D, MODE, SL>(p);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM (512 TMEM columns)
  cudaError_t e = cudaFuncSetAttribute(flash_dkdv_kernel<D, MODE, SL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if ((e = persistent_grid(prm.units, prm.counter, s, &grid)) != cudaSuccess) return e;
  if (grid == 0) return cudaSuccess;
  flash_dkdv_kernel<D, MODE, SL><<<grid, kBwThreads, smem, s>>>(mq, mo, mk, mv, prm);
  return cudaGetLastError();
}

cudaError_t launch_flash_dkdv(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const int mode = p.c.mode == SLA_MODE_THREEWAY ? kModeThree : p.c.nsa_branches ? kModeNsaTok : kModeTopn;
  if (p.c.d == 128) {
    if (mode == kModeNsaTok) return launch_dkdv_t<128, kModeNsaTok>(p, bp, a, s);
    return mode == kModeTopn ? launch_dkdv_t<128, kModeTopn>(p, bp, a, s) : launch_dkdv_t<128, kModeThree>(p, bp, a, s);
  }
  if (mode == kModeNsaTok) return launch_dkdv_t<64, kModeNsaTok>(p, bp, a, s);
  return mode == kModeTopn ? launch_dkdv_t<64, kModeTopn>(p, bp, a, s) : launch_dkdv_t<64, kModeThree>(p, bp, a, s);
}

cudaError_t launch_flash_dkdv_cmp(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  return p.c.d == 128 ? launch_dkdv_t<128, kModeNsaCmp>(p, bp, a, s) : launch_dkdv_t<64, kModeNsaCmp>(p, bp, a, s);
}

// ---------------------------------------------------------------------------
// NSA's compressed keys: dKc = scale * sum of the dK partials of a pair's chunks, dVc
// likewise, in chunk order (deterministic); rows past n_cmp are 0
// ---------------------------------------------------------------------------
__global__ void cmp_reduce_kernel(const float* __restrict__ part, float* __restrict__ dkc, float* __restrict__ dvc,
                                  CmpSplit sp, int items, int ncmp_pad, int d, int64_t total, float scale) {
  // one thread per (KV head, compressed key row, 4 columns)
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int q4 = d / 4;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += stride) {
    const int col = (int)(x % q4) * 4;
    const int64_t rowg = x / q4;
    const int row = (int)(rowg % ncmp_pad);
    const int64_t bkv = rowg / ncmp_pad;
    const int u = row / 128, r = row % 128;
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    if (row < sp.n_cmp) {
      int base = 0;
      for (int w = 0; w < u; ++w) base += sp.chunks(w);
      const int n = sp.chunks(u);
      for (int it = 0; it < n; ++it) {
        const float* pr = part + ((size_t)bkv * items + base + it) * 2 * 128 * d;
        const float4 v4 = *reinterpret_cast<const float4*>(pr + (size_t)r * d + col);
        const float4 k4 = *reinterpret_cast<const float4*>(pr + ((size_t)128 + r) * d + col);
        sv.x += v4.x; sv.y += v4.y; sv.z += v4.z; sv.w += v4.w;
        sk.x += k4.x; sk.y += k4.y; sk.z += k4.z; sk.w += k4.w;
      }
    }
    const size_t o = ((size_t)bkv * ncmp_pad + row) * d + col;
    *reinterpret_cast<float4*>(dvc + o) = sv;
    *reinterpret_cast<float4*>(dkc + o) = make_float4(scale * sk.x, scale * sk.y, scale * sk.z, scale * sk.w);
  }
}

cudaError_t launch_cmp_reduce(const Plan& p, const BwdPlan& bp, const BwdArgs& a, cudaStream_t s) {
  const sla_config& c = p.c;
  const int64_t total = (int64_t)c.B * c.H_kv * p.ncmp_pad * (c.d / 4);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  cmp_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      reinterpret_cast<const float*>(a.bws + bp.off_part), reinterpret_cast<float*>(a.bws + bp.off_dkc),
      reinterpret_cast<float*>(a.bws + bp.off_dvc), cmp_split(p), bp.cmp_items, p.ncmp_pad, c.d, total, p.scale);
  return cudaGetLastError();
}

}  // namespace sla
