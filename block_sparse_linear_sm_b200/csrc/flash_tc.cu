// Sparse exact attention over indexed key blocks on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
// 2025 sparse-attention review, section 2.3 (NSA operator design): load
// fixed-size indexed KV blocks, outer loop over queries, inner loop over the
// indexed KV blocks, filling the tensor cores. Three-way mode (SLA analysis
// page, arXiv 2509.24006): the blocks of a query block are its critical
// blocks. Top-n mode (2025 review section 4, MoBA; sparse attention survey
// section 2, NSA): the KV group's selected past blocks plus the blocks the
// causal window reaches; element (t, s) is kept when s <= t and (block(s) is
// selected or s > t - window).
//
// Work unit = 128 query rows = two halves of 64 rows:
//   - three-way mode, and top-n mode with an odd group size: query blocks
//     2p and 2p+1 of one head; their block lists are merged and a tile that
//     only one half needs is masked for the other half (such tiles of the two
//     halves alternate in the tile order, so both halves' warps stay busy);
//   - top-n mode with an even group size: two query heads of one KV group at
//     the same query block (identical lists, no masking waste).
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2-5 (one TMEM lane quarter each) run the online
// softmax, one thread per query row.
//
// Per tile n (64 keys): S_n = Q K_n^T (M=128, N=64) into one of two TMEM
// buffers; the softmax warps load S_n, mask and exponentiate it and write P_n
// (bf16, two per 32-bit column) back into the same TMEM buffer; O += P_n V_n
// (M=128, N=D, A read from TMEM) accumulates in TMEM. The MMA thread issues
// S_{n+2} into that buffer right after PV_n (tcgen05 operations of one thread
// execute in issue order), so two score tiles are always ahead of the softmax.
// The running max only moves (and O is rescaled) when a row's max grows by
// more than 2^8, so P stays below 256 and O needs no per-tile rescale.
//
// Shared memory: Q (128 x D bf16), a ring of three K slots (a K tile is free
// once S = Q K^T is done) and a ring of two V slots (free after P V), each
// refilled as soon as a slot frees, and the merged block list. Operand tiles use the 128-byte swizzle. Two CTAs fit on one SM
// (TMEM: 256 columns each).
#include "common.cuh"
#include "tc.cuh"

namespace sla {

struct FlashTcParams {
  const int32_t* list;  // THREEWAY: [B*H][nb][len] critical; TOPN: [B*H_kv][nb][len] selected (-1 pad)
  __nv_bfloat16* o;     // [B*H][N][D]
  int* status;
  int H, group, N, n_valid, nb, len, window;
  int pair_heads;       // 1: halves are heads (2hp, 2hp+1) of a group; 0: query blocks (2p, 2p+1)
  const float* zs;     // fused epilogue: Z_i [B*H][nqb][D] (fp32)
  const float* gate;   // fused epilogue: g_t = sigmoid(q_t . w_g[h]) [B*H][N] (fp32) or null
  float* lse;           // [B*H][N] row log2-sum-exp of the scaled scores (+inf: no key), or null
  int npairs;           // units per (b, h) when pairing query blocks
  int pair0;            // first pair of query blocks (pairing query blocks)
  int qb_first, qb_count;  // query blocks of the units (pairing heads)
  int words;            // 32-bit words of one block bitmap
  int list_cap;         // capacity of the merged list
  // Keys: n_keys valid keys in nkt 64-key tiles. Key index c stands for token
  // c * kstride + kspan in the causal test c * kstride + kspan <= t (1 and 0 for the
  // token keys; NSA's compressed keys: the stride and length - 1 of a compressed block).
  int n_keys, nkt, kstride, kspan;
  int dense_tiles;      // top-n mode: every key tile up to the causal limit (no list)
  float scale_log2;
  // NSA's window branch (NSAC): the compressed and selected branches' outputs [B*H][N][D]
  // and the branch gates w_g [H][3][D] (null: every gate is 1)
  const __nv_bfloat16* oc;
  const __nv_bfloat16* os;
  const __nv_bfloat16* w_g3;
  __nv_bfloat16* ow;  // NSAC: the window branch's own output o_w [B*H][N][D], kept for the backward pass
};

constexpr int kTcThreads = 192;
constexpr int kKSlots = 3;  // K tiles: freed as soon as S = Q K^T is done
constexpr int kVSlots = 2;  // V tiles: freed after P V
constexpr int kSlots = kKSlots + kVSlots;
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct TcLayout {
  static constexpr int kQBytes = 128 * D * 2;           // 2 halves x D/64 panels x 8 KB
  static constexpr int kSlotBytes = 64 * D * 2;         // one K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kSlotBytes;  // 32 mbarriers
  static constexpr int kOffMisc = kOffBar + 32 * 8;      // tmem addr, count, abort
  static constexpr int kOffList = kOffMisc + 64;         // merged block list
  static constexpr int kTmemCols = 256;                  // O: D columns, S: 2 x 64 columns
};

// FUSE (three-way layers with a linear branch): the epilogue of the layer runs
// in the kernel's tail. Once the last S and PV products are done, S'_i (tmS) and
// Z_i of both query blocks of the unit are loaded into the freed K/V rings and
// phi(Q) (tmF, written by the pooling pass) into the Q tiles; num = phi(Q) S'_i
// goes to the freed S columns of TMEM (one query block at a time) and
// O = O_s + g * num / (phi(q) . Z_i) is written to the output.
// KMAP (NSA's compressed branch only): key c stands for token c * kstride + kspan in the causal
// test, and the key tiles are every tile up to the causal limit (dense_tiles); compiled
// separately so that the plain top-n kernel keeps its registers.
// NSAC (NSA's window branch, the last of the three): the epilogue writes the layer's
// output O = g_c o_c + g_s o_s + g_w o_w, with this branch's o_w taken from TMEM in
// fp32, the other two read from the buffers the earlier launches wrote, and the gates
// g_b = sigmoid(q_t . w_g[h][b]) from the Q row still in shared memory.
template <int D, bool TOPN, bool FUSE, bool KMAP, bool NSAC = false>
__global__ void __launch_bounds__(kTcThreads, 2)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                    const __grid_constant__ CUtensorMap tmF, FlashTcParams prm) {
  using L = TcLayout<D>;
  constexpr int NP = D / 64;  // 64-column panels
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (sbase & 1023u) {  // swizzled operand tiles need 1024-byte alignment
    if (tid == 0) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashAlign);
    return;
  }

  // the four block bitmaps (act0, act1, sel0, sel1) and the union of the two
  // halves' blocks in block order only live during set-up, in the K/V ring before
  // its first load
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + L::kOffKV);
  uint32_t* mlist = reinterpret_cast<uint32_t*>(smem + L::kOffList);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] = TMEM base, misc[1] = merged count, misc[2] = abort
  auto bar = [&](int k) -> uint32_t { return sbase + L::kOffBar + 8 * k; };
  // barrier ids
  // barrier ids: K ring, V ring (full / empty per slot), S and P per TMEM buffer
  constexpr int Q_FULL = 0, K_FULL = 1, K_EMPTY = K_FULL + kKSlots, V_FULL = K_EMPTY + kKSlots,
                V_EMPTY = V_FULL + kVSlots, S_FULL = V_EMPTY + kVSlots, P_FULL = S_FULL + 2,
                O_DONE = P_FULL + 2, SP_FULL = O_DONE + 1, SP1_FULL = SP_FULL + 1, NUM_DONE = SP1_FULL + 1,
                NUM_READ = NUM_DONE + 4, O_LAST = NUM_READ + 1;
  // O_DONE completes once per P V product; O_LAST once, after the last one
  static_assert(O_LAST < 32, "barrier area holds 32 mbarriers");

  // ---- unit decode ----------------------------------------------------------
  const int Hkv = prm.H / prm.group;
  int bh_h[2], i_h[2], bkv;
  bool valid_h[2];
  const int32_t* lst[2];
  {
    const int u = blockIdx.x;
    if (!prm.pair_heads) {
      const int bh = u / prm.npairs, p = prm.pair0 + u % prm.npairs;
      const int b = bh / prm.H, h = bh % prm.H;
      bkv = b * Hkv + h / prm.group;
      for (int hf = 0; hf < 2; ++hf) {
        bh_h[hf] = bh;
        i_h[hf] = 2 * p + hf;
      }
    } else {
      const int hp_n = prm.group / 2;
      const int hp = u % hp_n;
      const int rest = u / hp_n;
      const int i = prm.qb_first + rest % prm.qb_count;
      bkv = rest / prm.qb_count;
      const int b = bkv / Hkv, g = bkv % Hkv;
      for (int hf = 0; hf < 2; ++hf) {
        bh_h[hf] = b * prm.H + g * prm.group + 2 * hp + hf;
        i_h[hf] = i;
      }
    }
    for (int hf = 0; hf < 2; ++hf) {
      valid_h[hf] = i_h[hf] < prm.nb;
      lst[hf] = nullptr;
      if (valid_h[hf] && prm.len > 0)
        lst[hf] = TOPN ? prm.list + ((size_t)bkv * prm.nb + i_h[hf]) * prm.len
                       : prm.list + ((size_t)bh_h[hf] * prm.nb + i_h[hf]) * prm.len;
    }
  }

  // ---- prologue: barriers, TMEM, merged block list --------------------------
  for (int w = tid; w < 4 * prm.words; w += kTcThreads) words[w] = 0u;
  if (tid == 0) {
    misc[2] = 0;
    tc::mbar_init(bar(Q_FULL), 1);
    for (int s = 0; s < kKSlots; ++s) {
      tc::mbar_init(bar(K_FULL + s), 1);
      tc::mbar_init(bar(K_EMPTY + s), 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      tc::mbar_init(bar(V_FULL + s), 1);
      tc::mbar_init(bar(V_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(S_FULL + b), 1);
      tc::mbar_init(bar(P_FULL + b), 4);
    }
    tc::mbar_init(bar(O_DONE), 1);
    tc::mbar_init(bar(O_LAST), 1);
    tc::mbar_init(bar(SP_FULL), 1);
    tc::mbar_init(bar(SP1_FULL), 1);
    for (int x = 0; x < 4; ++x) tc::mbar_init(bar(NUM_DONE + x), 1);  // (column pass, half)
    tc::mbar_init(bar(NUM_READ), 4);
    tc::fence_mbar_init();
    // Q does not depend on the block lists: its load overlaps the list merge
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
    tc::mbar_expect_tx(bar(Q_FULL), L::kQBytes);
    for (int hf = 0; hf < 2; ++hf)
      for (int p = 0; p < NP; ++p)
        tc::tma_load_3d(sbase + L::kOffQ + p * 16384 + hf * 8192, &tmQ, bar(Q_FULL), 64 * p,
                        i_h[hf] * kBlock, bh_h[hf]);
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + L::kOffMisc, L::kTmemCols);
    tc::tmem_relinquish();
  }
  __syncthreads();
  // bitmaps of the two halves
  for (int hf = 0; hf < 2; ++hf) {
    if (!valid_h[hf]) continue;
    uint32_t* act = words + hf * prm.words;
    uint32_t* sel = words + (2 + hf) * prm.words;
    for (int e = tid; e < prm.len; e += kTcThreads) {
      const int j = lst[hf][e];
      if (TOPN && j < 0) continue;  // padding of short selections
      if (j < 0 || j >= prm.nkt || (TOPN && j >= i_h[hf])) {
        report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashIndex);
        continue;
      }
      atomicOr(&act[j >> 5], 1u << (j & 31));
      if (TOPN) atomicOr(&sel[j >> 5], 1u << (j & 31));
    }
    if (TOPN && KMAP && prm.dense_tiles) {
      // every key tile with a key some row of this query block may attend
      const int last_t = i_h[hf] * kBlock + kBlock - 1 - prm.kspan;
      int jmax = last_t < 0 ? -1 : last_t / prm.kstride / kBlock;
      if (jmax > prm.nkt - 1) jmax = prm.nkt - 1;
      for (int j = tid; j <= jmax; j += kTcThreads) {
        atomicOr(&act[j >> 5], 1u << (j & 31));
        atomicOr(&sel[j >> 5], 1u << (j & 31));
      }
    }
    if (TOPN && prm.window > 0) {
      const int lo = i_h[hf] * kBlock - prm.window + 1;
      const int first = lo <= 0 ? 0 : lo / kBlock;
      for (int j = first + tid; j <= i_h[hf]; j += kTcThreads) atomicOr(&act[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    // the merge writes the union in block order into the free ring area after the
    // bitmaps; the reorder below moves it to mlist
    uint32_t* ulist = words + 4 * prm.words;
    int base = 0;
    for (int w0 = 0; w0 < prm.words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t a0 = w < prm.words ? words[w] : 0u, a1 = w < prm.words ? words[prm.words + w] : 0u;
      const uint32_t s0 = w < prm.words ? words[2 * prm.words + w] : 0u;
      const uint32_t s1 = w < prm.words ? words[3 * prm.words + w] : 0u;
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
        if (pos < prm.list_cap)
          ulist[pos] = (uint32_t)(w * 32 + bit) | ((a0 & m) ? 1u << 16 : 0u) | ((a1 & m) ? 1u << 17 : 0u) |
                       ((s0 & m) ? 1u << 18 : 0u) | ((s1 & m) ? 1u << 19 : 0u);
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int tm = base < prm.list_cap ? base : prm.list_cap;
    __syncwarp();
    // Tile order. A tile that only one half needs keeps the other half's warps idle
    // (they only store zero P rows), so such tiles of the two halves alternate: the
    // two halves' softmax warps then work on consecutive tiles at the same time (both
    // S buffers are in flight). The rest of the longer exclusive run follows, then the
    // tiles both halves need. Online softmax does not depend on the order.
    int n0 = 0, n1 = 0;
    for (int e0 = 0; e0 < tm; e0 += 32) {
      const int e = e0 + lane;
      const uint32_t v = e < tm ? ulist[e] : 0u;
      const bool a0 = (v >> 16) & 1u, a1 = (v >> 17) & 1u;
      n0 += __popc(__ballot_sync(0xffffffffu, e < tm && a0 && !a1));
      n1 += __popc(__ballot_sync(0xffffffffu, e < tm && a1 && !a0));
    }
    const int pairs = n0 < n1 ? n0 : n1, nex = n0 + n1;
    int r0 = 0, r1 = 0, rs = 0;
    const uint32_t below = (1u << lane) - 1u;
    for (int e0 = 0; e0 < tm; e0 += 32) {
      const int e = e0 + lane;
      const uint32_t v = e < tm ? ulist[e] : 0u;
      const bool a0 = (v >> 16) & 1u, a1 = (v >> 17) & 1u;
      const bool c0 = e < tm && a0 && !a1, c1 = e < tm && a1 && !a0, cs = e < tm && a0 && a1;
      const uint32_t b0 = __ballot_sync(0xffffffffu, c0), b1 = __ballot_sync(0xffffffffu, c1),
                     bs = __ballot_sync(0xffffffffu, cs);
      int pos = -1;
      if (c0) {
        const int r = r0 + __popc(b0 & below);
        pos = r < pairs ? 2 * r : pairs + r;
      } else if (c1) {
        const int r = r1 + __popc(b1 & below);
        pos = r < pairs ? 2 * r + 1 : pairs + r;
      } else if (cs) {
        pos = nex + rs + __popc(bs & below);
      }
      if (pos >= 0 && pos < tm) mlist[pos] = v;
      r0 += __popc(b0);
      r1 += __popc(b1);
      rs += __popc(bs);
    }
    if (lane == 0) {
      // every entry belongs to one of the three classes; anything else is a broken merge
      if (base > prm.list_cap || nex + rs != tm) report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashIndex);
      misc[1] = nex + rs == tm ? tm : 0;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int T = misc[1];
  const uint32_t tmem = (uint32_t)misc[0];
  volatile int* abort = misc + 2;
  const uint32_t sQ = sbase + L::kOffQ, sKV = sbase + L::kOffKV;

  if (warp == 0) {
    // ======================= TMA producer =====================================
    // without critical tiles nobody consumes Q: its load must still land before
    // the Q tiles are reused or the CTA exits
    if (lane == 0 && T == 0 && !tc::mbar_wait(bar(Q_FULL), 0, abort)) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
    if (lane == 0 && T > 0) {
      // K and V tiles go to separate rings; each is refilled as soon as a slot frees
      const uint32_t sKr = sKV, sVr = sKV + kKSlots * L::kSlotBytes;
      int nk = 0, nv = 0;
      uint64_t t0 = tc::globaltimer();
      uint32_t spins = 0;
      while (nk < T || nv < T) {
        bool progressed = false;
        if (nk < T && (nk < kKSlots || tc::mbar_test(bar(K_EMPTY + nk % kKSlots), ((nk / kKSlots) - 1) & 1))) {
          const int slot = nk % kKSlots, jb = (int)(mlist[nk] & 0xFFFFu);
          tc::mbar_expect_tx(bar(K_FULL + slot), L::kSlotBytes);
          for (int p = 0; p < NP; ++p)
            tc::tma_load_3d(sKr + slot * L::kSlotBytes + p * 8192, &tmK, bar(K_FULL + slot), 64 * p, jb * kBlock, bkv);
          ++nk;
          progressed = true;
        }
        if (nv < T && nv < nk && (nv < kVSlots || tc::mbar_test(bar(V_EMPTY + nv % kVSlots), ((nv / kVSlots) - 1) & 1))) {
          const int slot = nv % kVSlots, jb = (int)(mlist[nv] & 0xFFFFu);
          tc::mbar_expect_tx(bar(V_FULL + slot), L::kSlotBytes);
          for (int p = 0; p < NP; ++p)
            tc::tma_load_3d(sVr + slot * L::kSlotBytes + p * 8192, &tmV, bar(V_FULL + slot), 64 * p, jb * kBlock, bkv);
          ++nv;
          progressed = true;
        }
        if (progressed) {
          t0 = tc::globaltimer();
          spins = 0;
          continue;
        }
        __nanosleep(64);  // leave the issue slots to the softmax warp sharing this SMSP
        if ((++spins & 63u) == 0 && (*abort || tc::globaltimer() - t0 > tc::kTimeoutNs)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
          break;
        }
      }
      // tail: wait for the last release of every K slot (every S product done)
      for (int n = (T > kKSlots ? T - kKSlots : 0); n < nk && !*abort; ++n)
        if (!tc::mbar_wait(bar(K_EMPTY + n % kKSlots), (n / kKSlots) & 1, abort)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
        }
    }
    // Fused epilogue operands. The Q tiles and the K ring are free once every S
    // product is done: they take phi(Q), S'_i of the first query block and Z_i of
    // both, while the last P V products still run. S'_i of the second block goes
    // to the V ring after its last release.
    const int nh = valid_h[1] ? 2 : 1;
    if (FUSE && lane == 0 && !*abort) {
      tc::mbar_expect_tx(bar(SP_FULL), L::kQBytes + D * D * 2 + nh * D * 4);
      for (int hf = 0; hf < 2; ++hf)
        for (int p = 0; p < NP; ++p)
          tc::tma_load_3d(sQ + p * 16384 + hf * 8192, &tmF, bar(SP_FULL), 64 * p, i_h[hf] * kBlock,
                          bh_h[hf]);
      const int blk0 = bh_h[0] * prm.nb + i_h[0];
      for (int p = 0; p < NP; ++p)
        tc::tma_load_3d(sKV + p * D * 128, &tmS, bar(SP_FULL), 64 * p, 0, blk0);
      for (int hf = 0; hf < nh; ++hf)
        tc::bulk_load(sKV + D * D * 2 + hf * D * 4, prm.zs + (size_t)(bh_h[hf] * prm.nb + i_h[hf]) * D,
                      D * 4, bar(SP_FULL));
    }
    if (lane == 0 && T > 0) {
      // the last release of every V slot: no tcgen05.commit arrival is still in
      // flight when the CTA exits, and the V ring is free
      for (int n = (T > kVSlots ? T - kVSlots : 0); n < T && !*abort; ++n)
        if (!tc::mbar_wait(bar(V_EMPTY + n % kVSlots), (n / kVSlots) & 1, abort)) {
          *abort = 1;
          report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
        }
    }
    if (FUSE && lane == 0 && !*abort && nh == 2) {
      tc::mbar_expect_tx(bar(SP1_FULL), D * D * 2);
      const int blk1 = bh_h[1] * prm.nb + i_h[1];
      for (int p = 0; p < NP; ++p)
        tc::tma_load_3d(sKV + kKSlots * L::kSlotBytes + p * D * 128, &tmS, bar(SP1_FULL), 64 * p, 0, blk1);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    // The whole warp runs the loop (waits, descriptors); one elected lane issues.
    if (T > 0 || FUSE) {
      constexpr uint32_t kIdS = tc::idesc_bf16(128, 64, false, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(128, D, false, true);
      constexpr uint32_t kAll = 0xffffffffu;
      const uint32_t tO = tmem, tS0 = tmem + D;
      // base descriptors; a byte offset off is added as off >> 4 (start-address field)
      const uint64_t dQ = tc::sw128_desc(sQ, 16, 1024);
      const uint64_t dK = tc::sw128_desc(sKV, 16, 1024);
      const uint64_t dV = tc::sw128_desc(sKV + kKSlots * L::kSlotBytes, 8192, 1024);
      bool ok = T == 0 || __all_sync(kAll, tc::mbar_wait(bar(Q_FULL), 0, abort));
      tc::fence_after_sync();
      // S_n = Q K_n^T into TMEM buffer n & 1 (elected lane; K_n is resident)
      auto issue_s = [&](int n) {
        const int slot = n % kKSlots;
        const uint64_t dk = dK + (uint32_t)(slot * L::kSlotBytes >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_bf16_ss(tS0 + 64 * (n & 1), dQ + (uint32_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                          dk + (uint32_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4), kIdS, k > 0);
        tc::mma_commit(bar(S_FULL + (n & 1)));
        tc::mma_commit(bar(K_EMPTY + slot));
      };
      auto wait_k = [&](int n) -> bool {
        return __all_sync(kAll, tc::mbar_wait(bar(K_FULL + n % kKSlots), (n / kKSlots) & 1, abort));
      };
      for (int n = 0; n < 2 && n < T && ok; ++n) {
        ok = wait_k(n);
        tc::fence_after_sync();
        if (ok && tc::elect_one()) issue_s(n);
        __syncwarp();
      }
      for (int n = 0; n < T && ok; ++n) {
        const int b = n & 1, slot = n % kVSlots;
        // operands first (usually resident long before P_n is ready), then P_n
        ok = __all_sync(kAll, tc::mbar_wait(bar(V_FULL + slot), (n / kVSlots) & 1, abort)) &&
             (n + 2 >= T || wait_k(n + 2)) &&
             __all_sync(kAll, tc::mbar_wait(bar(P_FULL + b), (n >> 1) & 1, abort));
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t dv = dV + (uint32_t)(slot * L::kSlotBytes >> 4);
        if (tc::elect_one()) {
          // O += P_n V_n, A = P_n from TMEM buffer b
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_bf16_ts(tO, tS0 + 64 * b + 8 * kk, dv + (uint32_t)(kk * 2048 >> 4), kIdPV,
                            (n > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(bar(O_DONE));
          tc::mma_commit(bar(V_EMPTY + slot));
          if (n == T - 1) tc::mma_commit(bar(O_LAST));
          // buffer b is free once PV_n has read P_n: S_{n+2} goes in behind it
          // (tcgen05 operations of one thread execute in issue order)
          if (n + 2 < T) issue_s(n + 2);
        }
        __syncwarp();
      }
      if (FUSE && ok) {
        // num = phi(Q) S'_i into the 128 free S columns, 64 output columns per pass: half
        // hf's product (M = 128 rows, N = 64, K = D, B = S'_{i_hf}) goes to columns
        // 64 hf .. 64 hf + 63, so both halves' rows are ready together; the next pass
        // waits until all four softmax warps have read this one
        constexpr uint32_t kIdN = tc::idesc_bf16(128, 64, false, true);
        const uint64_t dS = tc::sw128_desc(sKV, D * 128, 1024);
        ok = __all_sync(kAll, tc::mbar_wait(bar(SP_FULL), 0, abort));
        for (int pass = 0; pass < D / 64 && ok; ++pass) {
          if (pass > 0) ok = __all_sync(kAll, tc::mbar_wait(bar(NUM_READ), (pass - 1) & 1, abort));
          for (int hf = 0; hf < 2 && ok; ++hf) {
            if (!valid_h[hf]) continue;
            if (pass == 0 && hf == 1) ok = __all_sync(kAll, tc::mbar_wait(bar(SP1_FULL), 0, abort));
            if (!ok) break;
            tc::fence_after_sync();
            if (tc::elect_one()) {
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
                tc::mma_bf16_ss(tS0 + 64 * hf, dQ + (uint32_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                                dS + (uint32_t)((hf * kKSlots * L::kSlotBytes + pass * D * 128 + k * 2048) >> 4),
                                kIdN, k > 0);
              tc::mma_commit(bar(NUM_DONE + 2 * pass + hf));
            }
            __syncwarp();
          }
        }
      }
      if (!ok && lane == 0) {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    }
  } else {
    // ======================= softmax warpgroup =================================
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;       // query row of the unit
    const int hf = r >> 6;
    const int t = i_h[hf] * kBlock + (r & 63);
    const int t_lo = i_h[hf] * kBlock + ((quarter * 32) & 63);  // first token of this warp
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off, tS0 = tmem + D + lane_off;
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY, l_sum = 0.f;    // m_ref in the scaled log2 domain
    bool ok = true;
    for (int n = 0; n < T; ++n) {
      const uint32_t e = mlist[n];
      const int jb = (int)(e & 0xFFFFu);
      const bool act = (e >> (16 + hf)) & 1u;   // uniform across the warp (one half per warp)
      const bool sel = (e >> (18 + hf)) & 1u;
      const int b = n & 1;
      const uint32_t tS = tS0 + 64 * b;
      // every lane takes the same branch: the TMEM accesses below are warp-collective
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar(S_FULL + b), (n >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t pk[32];
      float alpha = 1.f;
      bool resc = false;
      if (act) {
        uint32_t x0[32], x1[32];
        tc::tmem_ld32(tS, x0);
        tc::tmem_ld32(tS + 32, x1);
        tc::tmem_ld_wait();
        float x[64];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = __uint_as_float(x0[j]);
          x[32 + j] = __uint_as_float(x1[j]);
        }
        const int k0 = jb * kBlock;
        bool need_mask = k0 + kBlock > prm.n_keys;
        if (TOPN && KMAP)  // compressed keys: every tile counts as selected, no window
          need_mask = need_mask || (k0 + kBlock - 1) * prm.kstride + prm.kspan > t_lo;
        else if (TOPN)
          need_mask = need_mask || (k0 + kBlock - 1 > t_lo) || (!sel && k0 <= t_lo + 31 - prm.window);
        if (need_mask) {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const int key = k0 + j;
            bool keep = key < prm.n_keys;
            if (TOPN && KMAP)
              keep = keep && key * prm.kstride + prm.kspan <= t;
            else if (TOPN)
              keep = keep && key <= t && (sel || key > t - prm.window);
            x[j] = keep ? x[j] : -INFINITY;
          }
        }
        // row max with three-input max: 36 instructions for the 64 columns
        float mx[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(x[2 * u], x[2 * u + 1]);
#pragma unroll
        for (int j = 8; j < 32; ++j) mx[j & 7] = tc::fmax3(mx[j & 7], x[2 * j], x[2 * j + 1]);
        const float m_raw = tc::fmax3(tc::fmax3(mx[0], mx[1], mx[2]), tc::fmax3(mx[3], mx[4], mx[5]),
                                      fmaxf(mx[6], mx[7]));
        const float m_tile = m_raw * sl2;
        if (m_tile > m_ref + kRescaleLog2) {
          if (m_ref != -INFINITY) {
            alpha = tc::ex2_approx(m_ref - m_tile);
            resc = true;
          }
          m_ref = m_tile;
        }
        float psum = 0.f;
        if (m_ref != -INFINITY) {
          const uint64_t sc2 = tc::f2_pack(sl2, sl2), ng2 = tc::f2_pack(-m_ref, -m_ref);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const uint64_t y = tc::ffma2(tc::f2_pack(x[2 * j], x[2 * j + 1]), sc2, ng2);
            const float p0 = tc::ex2_approx(tc::f2_lo(y));
            const float p1 = tc::ex2_approx(tc::f2_hi(y));
            acc[j & 3] = tc::fadd2(acc[j & 3], tc::f2_pack(p0, p1));
            pk[j] = pack_bf16(p0, p1);
          }
          const uint64_t a2 = tc::fadd2(tc::fadd2(acc[0], acc[1]), tc::fadd2(acc[2], acc[3]));
          psum = tc::f2_lo(a2) + tc::f2_hi(a2);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) pk[j] = 0u;
        }
        l_sum = l_sum * alpha + psum;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = 0u;  // this half does not use the tile
      }
      // Only an O rescale waits for PV_{n-1} (it accumulates into O). P_n's buffer is free
      // without a wait: S_n went into it after PV_{n-2} had read P_{n-2} (one thread issues
      // both, in order). When this wait runs, the products PV_0 .. PV_{n-2} have completed
      // and PV_n has not been issued, so O_DONE has completed n - 1 or n phases and the
      // parity of phase n - 1 tells the two apart.
      const bool any_resc = __any_sync(0xffffffffu, resc);
      if (n > 0 && any_resc) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(bar(O_DONE), (n - 1) & 1, abort))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      if (any_resc) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tc::tmem_ld32(tO + 32 * c, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tc::tmem_st32(tO + 32 * c, ov);
        }
      }
      // P_n (bf16 pairs) into the first 32 columns of its S buffer
      tc::tmem_st32(tS, pk);
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(P_FULL + b));
    }
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(O_LAST), 0, abort));
      tc::fence_after_sync();
    }
    if (!ok) {
      *abort = 1;
      report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
    }
    // the backward pass recomputes P = 2^(s * scale * log2 e - lse) from this
    if (prm.lse != nullptr && valid_h[hf])
      prm.lse[(size_t)bh_h[hf] * prm.N + t] =
          (ok && T > 0 && l_sum > 0.f && t < prm.n_valid) ? m_ref + log2f(l_sum) : INFINITY;
    if (FUSE) {
      // ---- fused epilogue of the layer (three-way mode with a linear branch) ----
      // den = phi(q) . Z_i from the tiles the producer loaded (four partial sums)
      ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(SP_FULL), 0, abort));
      float den = 0.f;
      if (ok && valid_h[hf]) {
        const float4* z4 = reinterpret_cast<const float4*>(smem + L::kOffKV + D * D * 2 + hf * D * 4);
        float dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const uint4* frow = reinterpret_cast<const uint4*>(smem + L::kOffQ + p * 16384 + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 u = frow[c ^ (r & 7)];
            const float4 za = z4[16 * p + 2 * c], zb = z4[16 * p + 2 * c + 1];
            const float2 f0 = unpack_bf16(u.x), f1 = unpack_bf16(u.y), f2 = unpack_bf16(u.z),
                         f3 = unpack_bf16(u.w);
            dp[0] = fmaf(f0.x, za.x, fmaf(f0.y, za.y, dp[0]));
            dp[1] = fmaf(f1.x, za.z, fmaf(f1.y, za.w, dp[1]));
            dp[2] = fmaf(f2.x, zb.x, fmaf(f2.y, zb.y, dp[2]));
            dp[3] = fmaf(f3.x, zb.z, fmaf(f3.y, zb.w, dp[3]));
          }
        }
        den = (dp[0] + dp[1]) + (dp[2] + dp[3]);
      }
      const float g = (prm.gate && valid_h[hf] && t < prm.n_valid) ? prm.gate[(size_t)bh_h[hf] * prm.N + t] : 1.f;
      const float cl = den > 0.f ? g / den : 0.f;
      const bool live = ok && valid_h[hf] && t < prm.n_valid;
      const float inv = (live && T > 0 && l_sum > 0.f) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* og = prm.o + ((size_t)bh_h[hf] * prm.N + t) * D;
      // O = O_s / l + (g / den) num, 64 columns per pass of the num product
#pragma unroll 1
      for (int pass = 0; pass < D / 64; ++pass) {
        if (valid_h[hf]) {
          ok = ok && __all_sync(0xffffffffu, tc::mbar_wait(bar(NUM_DONE + 2 * pass + hf), 0, abort));
          tc::fence_after_sync();
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t ov[32], nv[32];
            if (ok) {
              if (T > 0) tc::tmem_ld32(tO + 64 * pass + 32 * c, ov);
              tc::tmem_ld32(tS0 + 64 * hf + 32 * c, nv);
              tc::tmem_ld_wait();
            }
            if (!ok || T == 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) ov[j] = 0u;
            }
            uint32_t pw[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pw[j] = live ? pack_bf16(__uint_as_float(ov[2 * j]) * inv + cl * __uint_as_float(nv[2 * j]),
                                       __uint_as_float(ov[2 * j + 1]) * inv + cl * __uint_as_float(nv[2 * j + 1]))
                           : 0u;
            uint4* dst = reinterpret_cast<uint4*>(og + 64 * pass + 32 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pw[4 * j], pw[4 * j + 1], pw[4 * j + 2], pw[4 * j + 3]);
          }
        }
        if (pass + 1 < D / 64) {
          // this pass's num columns are read (every softmax warp arrives, with or without
          // a valid half): the next pass may overwrite them
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(bar(NUM_READ));
        }
      }
      if (!ok) {
        *abort = 1;
        report(prm.status, SLA_ERR_DEVICE_TIMEOUT, kDetailTimeout);
      }
    } else if (NSAC && valid_h[hf]) {
      // NSA's gated sum of the three branches; padding rows are zero
      const bool live = ok && t < prm.n_valid;
      const float inv = (live && T > 0 && l_sum > 0.f) ? 1.f / l_sum : 0.f;
      float g[3] = {1.f, 1.f, 1.f};
      if (prm.w_g3 != nullptr && live) {
        const __nv_bfloat16* wg = prm.w_g3 + (size_t)(bh_h[hf] % prm.H) * 3 * D;
        float dot[3] = {0.f, 0.f, 0.f};
#pragma unroll 1
        for (int p = 0; p < NP; ++p) {
          const uint4* qrow = reinterpret_cast<const uint4*>(smem + L::kOffQ + p * 16384 + r * 128);
#pragma unroll 2
          for (int c = 0; c < 8; ++c) {
            const uint4 u = qrow[c ^ (r & 7)];
            const uint32_t uq[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int b = 0; b < 3; ++b) {
              const uint4 w = __ldg(reinterpret_cast<const uint4*>(wg + (size_t)b * D + p * 64 + c * 8));
              const uint32_t uw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 fq = unpack_bf16(uq[e]), fw = unpack_bf16(uw[e]);
                dot[b] = fmaf(fq.x, fw.x, fmaf(fq.y, fw.y, dot[b]));
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < 3; ++b) g[b] = 1.f / (1.f + __expf(-dot[b]));
      }
      const size_t rowoff = ((size_t)bh_h[hf] * prm.N + t) * D;
      const uint4* oc4 = reinterpret_cast<const uint4*>(prm.oc + rowoff);
      const uint4* os4 = reinterpret_cast<const uint4*>(prm.os + rowoff);
      uint4* dst = reinterpret_cast<uint4*>(prm.o + rowoff);
      uint4* dstw = reinterpret_cast<uint4*>(prm.ow + rowoff);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (ok && T > 0) {
          tc::tmem_ld32(tO + 32 * c, ov);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = 0u;
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 res = make_uint4(0u, 0u, 0u, 0u), resw = res;
          if (live) {
            const uint4 a4 = oc4[4 * c + q8], b4 = os4[4 * c + q8];
            const uint32_t ua[4] = {a4.x, a4.y, a4.z, a4.w}, ub[4] = {b4.x, b4.y, b4.z, b4.w};
            uint32_t pw[4], ww[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 fa = unpack_bf16(ua[e]), fb = unpack_bf16(ub[e]);
              const int j = 8 * q8 + 2 * e;
              const float w0 = __uint_as_float(ov[j]) * inv, w1 = __uint_as_float(ov[j + 1]) * inv;
              pw[e] = pack_bf16(g[0] * fa.x + g[1] * fb.x + g[2] * w0, g[0] * fa.y + g[1] * fb.y + g[2] * w1);
              ww[e] = pack_bf16(w0, w1);
            }
            res = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            resw = make_uint4(ww[0], ww[1], ww[2], ww[3]);
          }
          dst[4 * c + q8] = res;
          dstw[4 * c + q8] = resw;
        }
      }
    } else if (valid_h[hf]) {
      // epilogue: O / l -> bf16 rows (padding tokens and empty rows are zero)
      const float inv = (ok && T > 0 && l_sum > 0.f && t < prm.n_valid) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* og = prm.o + ((size_t)bh_h[hf] * prm.N + t) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (ok && T > 0) {
          tc::tmem_ld32(tO + 32 * c, ov);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = 0u;
        }
        uint32_t pw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pw[j] = inv == 0.f ? 0u
                             : pack_bf16(__uint_as_float(ov[2 * j]) * inv, __uint_as_float(ov[2 * j + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(og + 32 * c);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pw[4 * j], pw[4 * j + 1], pw[4 * j + 2], pw[4 * j + 3]);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// 3D map over [heads][rows][D] bf16: rows beyond n_rows read as zero; box 64 x 64 x 1.
static bool make_map(CUtensorMap* m, const void* base, int heads, int n_rows, int N, int D) {
  return make_tmap_3d(m, base, (uint64_t)D, (uint64_t)n_rows, (uint64_t)heads, (uint64_t)D * 2,
                      (uint64_t)N * D * 2, 64, 64);
}

// branch 0: the layer's sparse branch. NSA's branches (top-n mode with nsa_branches), each
// written to its own buffer: 1 compressed (keys: the compressed K, V; every tile up to the
// causal limit), 2 selected (the selected blocks only), 3 window (the window only).
template <int D, bool TOPN, bool FUSE, bool KMAP = false, bool NSAC = false>
static cudaError_t launch_tc(const Plan& p, const Args& a, int branch, cudaStream_t s) {
  using L = TcLayout<D>;
  const sla_config& c = p.c;
  const bool cmp = branch == 1;
  CUtensorMap mq, mk, mv, ms;
  const void* kb = cmp ? (const void*)(a.ws + p.off_kc) : (const void*)a.k;
  const void* vb = cmp ? (const void*)(a.ws + p.off_vc) : (const void*)a.v;
  const int key_rows = cmp ? (p.n_cmp > 0 ? p.n_cmp : 1) : c.N_valid, key_stride_rows = cmp ? p.ncmp_pad : c.N;
  if (!make_map(&mq, a.q, c.B * c.H, c.N_valid, c.N, D) ||
      !make_map(&mk, kb, c.B * c.H_kv, key_rows, key_stride_rows, D) ||
      !make_map(&mv, vb, c.B * c.H_kv, key_rows, key_stride_rows, D))
    return cudaErrorInvalidValue;
  // phi(Q) from the pooling pass, same geometry as Q (fused epilogue); otherwise unused
  CUtensorMap mf;
  if (!make_map(&mf, FUSE ? (const void*)(a.ws + p.off_phiq) : (const void*)a.q, c.B * c.H, c.N_valid, c.N, D))
    return cudaErrorInvalidValue;
  // S'_i as [B*H*nqb][D rows][D columns], box 64 x D (fused epilogue); otherwise unused
  if (!make_tmap_3d(&ms, FUSE ? (const void*)(a.ws + p.off_ss) : (const void*)a.q, D, D,
                    FUSE ? (uint64_t)c.B * c.H * p.nqb : 1, (uint64_t)D * 2, (uint64_t)D * D * 2, 64, D))
    return cudaErrorInvalidValue;
  FlashTcParams prm;
  prm.list = a.crit;
  // the sparse branch is the output, or the fused epilogue writes it; NSA's branches
  // each write their own buffer
  // NSA's window branch (the last) writes the gated sum of the three into the output
  prm.o = (branch == 0 || branch == 3) ? a.out
                                       : reinterpret_cast<__nv_bfloat16*>(a.ws + (branch == 1 ? p.off_oc : p.off_os));
  prm.oc = branch == 3 ? reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_oc) : nullptr;
  prm.os = branch == 3 ? reinterpret_cast<const __nv_bfloat16*>(a.ws + p.off_os) : nullptr;
  prm.w_g3 = branch == 3 && c.has_gate ? a.w_g : nullptr;
  prm.zs = FUSE ? reinterpret_cast<const float*>(a.ws + p.off_zs) : nullptr;
  prm.gate = FUSE && c.has_gate ? reinterpret_cast<const float*>(a.ws + p.off_gate) : nullptr;
  // row log-sum-exp for the backward pass; NSA's branches keep one row each
  // (compressed, selected, window)
  prm.lse = reinterpret_cast<float*>(a.ws + p.off_lse) + (branch > 0 ? (size_t)(branch - 1) * c.B * c.H * c.N : 0);
  prm.ow = branch == 3 ? reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_ow) : nullptr;
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = p.nkb;
  prm.len = (branch == 1 || branch == 3) ? 0 : (TOPN ? c.top_n : c.k_h);
  prm.window = (branch == 1 || branch == 2) ? 0 : c.window;
  prm.pair_heads = TOPN && (p.group % 2 == 0);
  // the query blocks [qb0, qb1) of the call: pairs qb0 / 2 .. (qb1 + 1) / 2 - 1
  prm.pair0 = p.qb0 / 2;
  prm.npairs = (p.qb1 + 1) / 2 - p.qb0 / 2;
  prm.qb_first = p.qb0;
  prm.qb_count = p.qb1 - p.qb0;
  prm.n_keys = cmp ? p.n_cmp : c.N_valid;
  prm.nkt = cmp ? p.ncmp_pad / kBlock : p.nkb;
  prm.kstride = cmp ? c.cmp_stride : 1;
  prm.kspan = cmp ? c.cmp_block - 1 : 0;
  prm.dense_tiles = cmp ? 1 : 0;
  prm.words = (prm.nkt + 31) / 32;
  int per_half = prm.len;
  if (TOPN) per_half += (prm.window + 62) / kBlock + 2;
  prm.list_cap = 2 * per_half < prm.nkt ? 2 * per_half : prm.nkt;
  if (cmp) prm.list_cap = prm.nkt;
  if (prm.list_cap < 1) prm.list_cap = 1;
  prm.scale_log2 = p.scale * 1.4426950408889634f;
  int smem = L::kOffList + prm.list_cap * 4;
  // the set-up bitmaps and the block-order union live in the ring before its first load
  if ((4 * prm.words + prm.list_cap) * 4 > kSlots * L::kSlotBytes) return cudaErrorInvalidValue;
  // at most two CTAs per SM: each holds 256 of the SM's 512 TMEM columns
  if (smem < 80 * 1024) smem = 80 * 1024;
  cudaError_t e = cudaFuncSetAttribute(flash_tc_kernel<D, TOPN, FUSE, KMAP, NSAC>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int units;
  if (prm.pair_heads)
    units = c.B * c.H_kv * prm.qb_count * (p.group / 2);
  else
    units = c.B * c.H * prm.npairs;
  flash_tc_kernel<D, TOPN, FUSE, KMAP, NSAC><<<units, kTcThreads, smem, s>>>(mq, mk, mv, ms, mf, prm);
  return cudaGetLastError();
}

cudaError_t launch_flash(const Plan& p, const Args& a, cudaStream_t s) {
  const bool topn = p.c.mode == SLA_MODE_TOPN_WINDOW;
  // the layer has a linear branch: marginal blocks, or every block with linear_all
  const bool fuse = !topn && (p.nkb - p.c.k_h - p.c.k_l > 0 || p.c.linear_all);
  if (p.c.d == 128) {
    if (topn) return launch_tc<128, true, false>(p, a, 0, s);
    return fuse ? launch_tc<128, false, true>(p, a, 0, s) : launch_tc<128, false, false>(p, a, 0, s);
  }
  if (topn) return launch_tc<64, true, false>(p, a, 0, s);
  return fuse ? launch_tc<64, false, true>(p, a, 0, s) : launch_tc<64, false, false>(p, a, 0, s);
}

cudaError_t launch_flash_nsa(const Plan& p, const Args& a, int branch, cudaStream_t s) {
  if (branch == 1)  // compressed keys: the key-to-token map and the dense tile range
    return p.c.d == 128 ? launch_tc<128, true, false, true>(p, a, branch, s)
                        : launch_tc<64, true, false, true>(p, a, branch, s);
  if (branch == 3)  // the window branch, with the gated sum of the three branches
    return p.c.d == 128 ? launch_tc<128, true, false, false, true>(p, a, branch, s)
                        : launch_tc<64, true, false, false, true>(p, a, branch, s);
  return p.c.d == 128 ? launch_tc<128, true, false>(p, a, branch, s) : launch_tc<64, true, false>(p, a, branch, s);
}

}  // namespace sla
