// Sparse exact attention over indexed key blocks.
//
// 2025 sparse-attention review, section 2.3 (NSA operator design): load
// fixed-size indexed KV blocks, outer loop over query blocks, inner loop over
// the indexed KV blocks. Each CTA owns one (b, h, query block i) and walks its
// block list with an online softmax (FlashAttention-style, fp32 statistics).
//
// Three-way mode: the list is the row's critical blocks; only key padding is
// masked. Top-n mode: the list is the KV group's selected past blocks merged
// with the blocks the causal window reaches; element (t, s) is kept when
// s <= t and (block(s) is selected or s > t - window).
#include "common.cuh"

namespace sla {

struct FlashParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o;        // [B*H][N][D]
  const int32_t* list;     // THREEWAY: [B*H][nb][len]; TOPN: [B*H_kv][nb][len]
  int* status;
  int H, group, N, n_valid, nb, len, window;
  float scale_log2;        // softmax scale * log2(e)
};

constexpr int kFlashThreads = 128;
constexpr int kMaxUnion = 128;  // selected blocks + window blocks (checked on the host)

template <int D, bool TOPN>
__global__ void __launch_bounds__(kFlashThreads) flash_kernel(FlashParams prm) {
  constexpr int RB = D * 2, CH = D / 8;
  constexpr int TILE = kBlock * RB;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* q_s = smem;
  unsigned char* k_s = smem + TILE;          // 2 buffers
  unsigned char* v_s = smem + 3 * TILE;      // 2 buffers
  __shared__ int blist[kMaxUnion];
  __shared__ int bcount;

  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / prm.H, h = bh % prm.H;
  const int bkv = b * (prm.H / prm.group) + h / prm.group;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const __nv_bfloat16* qg = prm.q + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
  const __nv_bfloat16* kg = prm.k + (size_t)bkv * prm.N * D;
  const __nv_bfloat16* vg = prm.v + (size_t)bkv * prm.N * D;

  // ---- block list ----------------------------------------------------------
  const int32_t* lrow;
  int count;
  if (!TOPN) {
    lrow = prm.list + ((size_t)bh * prm.nb + i) * prm.len;
    count = prm.len;
  } else {
    if (tid == 0) {
      const int32_t* sel = prm.list + ((size_t)bkv * prm.nb + i) * prm.len;
      int first_win = i + 1;
      if (prm.window > 0) {
        int lo = i * kBlock - prm.window + 1;
        first_win = lo <= 0 ? 0 : lo / kBlock;
      }
      // merge the ascending selected list (all < i, -1 padded) with the window
      // blocks [first_win, i]; bit 30 marks a selected block
      int n = 0, u = 0;
      while (u < prm.len && sel[u] >= 0 && sel[u] < first_win && n < kMaxUnion)
        blist[n++] = sel[u++] | (1 << 30);
      for (int jb = first_win; jb <= i && n < kMaxUnion; ++jb) {
        const bool s = u < prm.len && sel[u] == jb;
        if (s) ++u;
        blist[n++] = jb | (s ? (1 << 30) : 0);
      }
      bcount = n;
    }
    __syncthreads();
    lrow = nullptr;
    count = bcount;
  }
  auto block_at = [&](int n) -> int {
    int jb = TOPN ? (blist[n] & ~(1 << 30)) : lrow[n];
    if (jb < 0 || jb >= prm.nb) {
      report(prm.status, SLA_ERR_DEVICE_CHECK, kDetailFlashIndex);
      jb = -1;
    }
    return jb;
  };

  const uint32_t q_base = smem_u32(q_s), k_base = smem_u32(k_s), v_base = smem_u32(v_s);
  auto load_kv = [&](int buf, int jb) {
    const int nvk = min(kBlock, prm.n_valid - jb * kBlock);
    for (int e = tid; e < kBlock * CH; e += kFlashThreads) {
      const int t = e / CH, ch = e % CH;
      const size_t off = ((size_t)jb * kBlock + t) * D + ch * 8;
      const int bytes = t < nvk ? 16 : 0;
      cp_async16(k_base + buf * TILE + swz(t, ch, RB), kg + (bytes ? off : 0), bytes);
      cp_async16(v_base + buf * TILE + swz(t, ch, RB), vg + (bytes ? off : 0), bytes);
    }
  };

  // Q tile (padding rows read as zero)
  {
    const int nvq = min(kBlock, prm.n_valid - i * kBlock);
    for (int e = tid; e < kBlock * CH; e += kFlashThreads) {
      const int t = e / CH, ch = e % CH;
      const int bytes = t < nvq ? 16 : 0;
      cp_async16(q_base + swz(t, ch, RB), qg + (bytes ? (size_t)t * D + ch * 8 : 0), bytes);
    }
  }
  int cur = count > 0 ? block_at(0) : -1;
  if (cur >= 0) load_kv(0, cur);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int row0 = 16 * w + (lane >> 2);           // this thread's rows: row0, row0 + 8
  const int t_row[2] = {i * kBlock + row0, i * kBlock + row0 + 8};

  for (int n = 0; n < count; ++n) {
    const int jb = cur;
    const bool sel_blk = TOPN ? ((blist[n] >> 30) & 1) : true;
    cp_async_wait<0>();
    __syncthreads();
    if (n + 1 < count) {
      cur = block_at(n + 1);
      if (cur >= 0) load_kv((n + 1) & 1, cur);
    }
    cp_async_commit();
    if (jb < 0) continue;
    const uint32_t kb = k_base + (n & 1) * TILE, vb = v_base + (n & 1) * TILE;

    // S = Q K^T for 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int x = 0; x < 8; ++x) s[x][0] = s[x][1] = s[x][2] = s[x][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(lds_a(q_base, 16 * w, 2 * ks, RB, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(lds_b_nk(kb, n2 * 16, 2 * ks, RB, lane), b0, b1, b2, b3);
        mma_bf16(s[2 * n2], a, b0, b1);
        mma_bf16(s[2 * n2 + 1], a, b2, b3);
      }
    }
    // mask, scale to log2 domain, row max
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int x = 0; x < 8; ++x) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = jb * kBlock + x * 8 + 2 * (lane & 3) + (e & 1);
        const int rr = e >> 1;
        bool ok = key < prm.n_valid;
        if (TOPN) ok = ok && key <= t_row[rr] && (sel_blk || key > t_row[rr] - prm.window);
        const float val = ok ? s[x][e] * prm.scale_log2 : -INFINITY;
        s[x][e] = val;
        mx[rr] = fmaxf(mx[rr], val);
      }
    }
    float alpha[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
      const float m_new = fmaxf(m_r[rr], mx[rr]);
      alpha[rr] = m_new == -INFINITY ? 1.f : exp2f(m_r[rr] - m_new);
      m_r[rr] = m_new;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int x = 0; x < 8; ++x) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rr = e >> 1;
        const float p = m_r[rr] == -INFINITY ? 0.f : exp2f(s[x][e] - m_r[rr]);
        s[x][e] = p;
        rs[rr] += p;
      }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) l_r[rr] = l_r[rr] * alpha[rr] + rs[rr];
#pragma unroll
    for (int d8 = 0; d8 < D / 8; ++d8) {
      o[d8][0] *= alpha[0];
      o[d8][1] *= alpha[0];
      o[d8][2] *= alpha[1];
      o[d8][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int d2 = 0; d2 < D / 16; ++d2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(lds_b_kn(vb, kk * 16, 2 * d2, RB, lane), b0, b1, b2, b3);
        mma_bf16(o[2 * d2], a, b0, b1);
        mma_bf16(o[2 * d2 + 1], a, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  // row sums across the 4 lanes of a row, normalise, store
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 1);
    l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 2);
  }
  const float inv0 = (l_r[0] > 0.f && t_row[0] < prm.n_valid) ? 1.f / l_r[0] : 0.f;
  const float inv1 = (l_r[1] > 0.f && t_row[1] < prm.n_valid) ? 1.f / l_r[1] : 0.f;
  __nv_bfloat16* og = prm.o + ((size_t)bh * prm.N + (size_t)i * kBlock) * D;
#pragma unroll
  for (int d8 = 0; d8 < D / 8; ++d8) {
    const int col = d8 * 8 + 2 * (lane & 3);
    *reinterpret_cast<uint32_t*>(og + (size_t)row0 * D + col) =
        pack_bf16(o[d8][0] * inv0, o[d8][1] * inv0);
    *reinterpret_cast<uint32_t*>(og + (size_t)(row0 + 8) * D + col) =
        pack_bf16(o[d8][2] * inv1, o[d8][3] * inv1);
  }
}

template <int D, bool TOPN>
static cudaError_t launch_flash_t(const Plan& p, const Args& a, cudaStream_t s) {
  const sla_config& c = p.c;
  FlashParams prm;
  prm.q = a.q;
  prm.k = a.k;
  prm.v = a.v;
  prm.o = TOPN ? a.out : reinterpret_cast<__nv_bfloat16*>(a.ws + p.off_os);
  prm.list = a.crit;
  prm.status = a.status;
  prm.H = c.H;
  prm.group = p.group;
  prm.N = c.N;
  prm.n_valid = c.N_valid;
  prm.nb = p.nkb;
  prm.len = TOPN ? c.top_n : c.k_h;
  prm.window = c.window;
  prm.scale_log2 = p.scale * 1.4426950408889634f;
  const int smem = 5 * kBlock * D * 2;
  cudaError_t e = cudaFuncSetAttribute(flash_kernel<D, TOPN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nqb, c.B * c.H);
  flash_kernel<D, TOPN><<<grid, kFlashThreads, smem, s>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_flash(const Plan& p, const Args& a, cudaStream_t s) {
  const bool topn = p.c.mode == SLA_MODE_TOPN_WINDOW;
  if (p.c.d == 128) return topn ? launch_flash_t<128, true>(p, a, s) : launch_flash_t<128, false>(p, a, s);
  return topn ? launch_flash_t<64, true>(p, a, s) : launch_flash_t<64, false>(p, a, s);
}

}  // namespace sla
