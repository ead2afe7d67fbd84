// Index-based block-sparse attention over routed 128-token KV tiles.
//
// Digest of arXiv 2610.22311, "Core method" (Eq. 15) and "Novelty"; Velox
// project page, "Why the route is a block, not a token": the kernel visits
// only the KV tiles listed in a query block's route, so a skipped tile saves
// both its QK^T product and its K/V load.  The result is an ordinary softmax
// attention restricted to the tokens of the listed tiles, computed with the
// FlashAttention online-softmax recurrence over tiles.
//
// sm_100a design: one CTA per (head, query block), one CTA per SM.  The
// tiles of the route are split into two interleaved chains, even and odd,
// each with its own S buffer and its own O accumulator in TMEM (4 x 128
// columns) and its own softmax warpgroup with its own running max and row
// sum, so two tiles are in their softmax at once; the epilogue merges the
// two partial results (FlashAttention's split-KV merge, inside the CTA).
// CTAs take rows in the order `row_order` gives (longest routes first, from
// velox_route_schedule), so the last wave is made of short rows.
//   warp 0      TMA producer: Q once, then K_0, V_0, K_1, V_1, ... of the
//               route into a ring of 32 KB slots (128-byte swizzle, two
//               64-channel boxes per tile).
//   warp 1      TMEM allocator and the single tcgen05.mma issuer.  S_j =
//               Q K_j^T (both operands from shared memory) goes into buffer
//               j mod 2; once the softmax of tile j is done it issues
//               O_{j mod 2} += P_j V_j (A = P from TMEM, B = V from shared
//               memory) and, as soon as that has completed, S_{j+2} into the
//               same buffer.
//   warps 2-5   softmax of the even tiles, warps 6-9 of the odd tiles: one
//               query row per thread (its TMEM lane).  Two TMEM reads of the
//               S row (168 registers per thread do not hold the row and the
//               rest): the three-input max, then 32 columns at a time the
//               scaled exponent arguments and the row sum in packed fp32x2
//               arithmetic, exponentials on MUFU,
//               P_j packed to bf16 into the first 64 columns of its own S
//               buffer (column t/2 holds elements t, t+1).  A chain's running
//               max only moves (and its O is rescaled in TMEM, after its
//               previous PV) when it grows by more than 2^8; a stale max is
//               exact because the chain's O and row sum use the same one.
//               Epilogue: the two chains exchange (max, sum) per row through
//               shared memory; thread (row, chain c) writes channels
//               64c..64c+63 of O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / l, and lse.
// A pre-pass compacts the route into shared memory, skipping ids outside
// [0, M) and repeats (flagged in dev_status).
//
// Two-phase form (digest, "Reproducibility": the two-phase tile loop): after
// the routed history tiles the same loop visits the n_cur tiles of the
// current chunk's own K/V (separate tensors), alternating between the two
// chains like any other tiles, so the merged normaliser covers both phases.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace velox {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // tokens per KV tile
constexpr int D = 128;   // head dim
constexpr int kThreads = 320;  // TMA warp, MMA warp, 2 x 4 softmax warps
constexpr int kChainThreads = 128;  // softmax threads of one chain
constexpr int kSoftThreads = 256;
constexpr uint32_t kTileBytes = BN * D * 2;      // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-channel box
constexpr int kMaxRoute = VELOX_MAX_ROUTE;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBufs = 2;         // S/P buffers in TMEM (one per chain), columns 0 and 128
constexpr uint32_t kColO = 256;   // O accumulators (fp32, 128 columns each), 256 and 384
constexpr int kMaxSlots = 6;      // K/V ring slots of 32 KB
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest tolerated growth

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffRing = kOffQ + kTileBytes;
// barriers, misc and the dynamic tail follow the ring (offset set at launch)
// q_full, the K/V ring, s_full/p_full/pv_done per chain, x_fin, mma_done
constexpr uint32_t kNumBars = 1 + 2 * kMaxSlots + 3 * kSBufs + 1 + 1;
constexpr uint32_t kMiscBytes = 64;
constexpr uint32_t kSmemLimit = 227 * 1024;

struct AttnArgs {
  const uint16_t *Q;         // [H][N * 128][128] bf16
  const int32_t *route_ids;  // null: dense
  const int32_t *route_len;
  const int32_t *row_order;  // null: row = blockIdx.x
  int R_max;
  int N, M;
  int rows;                  // H * N
  int n_cur;                 // current-chunk tiles after the routed ones (0: none)
  float scale_log2;  // softmax_scale * log2(e)
  uint16_t *O;
  float *lse;
  int32_t *dev_status;
  int nslot;              // K/V ring slots in use (4..kMaxSlots)
  uint32_t bar_offset;    // byte offset of the barriers from the aligned base
  uint32_t list_offset;   // route list (uint16)
  uint32_t bits_offset;   // id bitmap (uint32)
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int k) {
  // K-major operand, 128-byte swizzle: 16-element K steps advance 32 bytes
  // inside a 64-element atom; atoms (64 channels) are 16 KB apart.
  return smem_desc_sw128(tile_saddr + (k >> 2) * kHalfBytes + (k & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t vmn_desc(uint32_t tile_saddr, int k) {
  // V as the MN-major B operand (N = channel, K = token): 16-token K steps
  // advance 16 rows of 128 bytes; the two 64-channel halves are 16 KB apart.
  return smem_desc_sw128(tile_saddr + k * 16 * 128, kHalfBytes, 1024);
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A (P, bf16) read from TMEM.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-uniform bounded wait (tcgen05.ld/st after it are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// 10 warps: three share a scheduler, whose 16 K registers then allow 168 each
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = base + kOffQ;
  uint8_t *ring = base + kOffRing;
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + a.bar_offset);
  uint64_t *q_full = bar;
  uint64_t *slot_full = q_full + 1;
  uint64_t *slot_empty = slot_full + kMaxSlots;
  uint64_t *s_full = slot_empty + kMaxSlots;   // [chain]
  uint64_t *p_full = s_full + kSBufs;          // [chain]
  uint64_t *pv_done = p_full + kSBufs;         // [chain]
  uint64_t *x_fin = pv_done + kSBufs;          // both chains' (max, sum) written
  uint64_t *mma_done = x_fin + 1;
  uint8_t *misc = base + a.bar_offset + kNumBars * 8;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(misc);
  int *s_nvalid = reinterpret_cast<int *>(misc + 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(misc + 8);
  uint16_t *tiles = reinterpret_cast<uint16_t *>(base + a.list_offset);
  uint32_t *bits = reinterpret_cast<uint32_t *>(base + a.bits_offset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = a.row_order ? a.row_order[blockIdx.x] : (int)blockIdx.x;
  if (row < 0 || row >= a.rows) {  // same value in every thread: uniform exit
    if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_BAD_ROW_ORDER);
    return;
  }
  const int h = row / a.N, i = row - h * a.N;
  const bool dense = (a.route_ids == nullptr);
  const int M = a.M;
  const int nslot = a.nslot;

  // ---- set-up: barriers, TMEM, route compaction
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kMaxSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kChainThreads);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(x_fin, kSoftThreads);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  int L = 0;
  if (!dense) {
    L = a.route_len[row];
    if (L < 0 || L > a.R_max) {
      if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_ROUTE_LEN);
      L = 0;
    }
    const int W = (M + 31) >> 5;
    for (int k = threadIdx.x; k < W; k += kThreads) bits[k] = 0u;
  }
  __syncthreads();
  if (warp == 0) {
    if (dense) {
      if (lane == 0) *s_nvalid = M;
    } else {
      const int32_t *ids = a.route_ids + (size_t)row * a.R_max;
      int n = 0;
      bool bad = false, dup = false;
      for (int b0 = 0; b0 < L; b0 += 32) {
        const int j = b0 + lane;
        const int id = j < L ? ids[j] : -1;
        bool ok = (j < L) && id >= 0 && id < M;
        if (j < L && !ok) bad = true;
        if (ok) {
          const uint32_t m = 1u << (id & 31);
          if (atomicOr(&bits[id >> 5], m) & m) {
            ok = false;
            dup = true;
          }
        }
        const unsigned vote = __ballot_sync(0xffffffffu, ok);
        if (ok) tiles[n + __popc(vote & ((1u << lane) - 1u))] = static_cast<uint16_t>(id);
        n += __popc(vote);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) flag_error(a.dev_status, VELOX_DEV_BAD_ROUTE_ID);
      if (__any_sync(0xffffffffu, dup) && lane == 0) flag_error(a.dev_status, VELOX_DEV_DUP_ROUTE_ID);
      if (lane == 0) *s_nvalid = n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n_hist = *s_nvalid;
  const int n = n_hist + a.n_cur;  // tiles of both phases
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (a.n_cur > 0) {
        prefetch_tmap(&tmKc);
        prefetch_tmap(&tmVc);
      }
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_3d(sQ, &tmQ, q_full, 0, i * BM, h);
      tma_load_3d(sQ + kHalfBytes, &tmQ, q_full, 64, i * BM, h);
      int issued = 0;
      for (int li = 0; li < 2 * n; ++li) {  // load li: K_{li/2} (even) or V_{li/2} (odd)
        const int s = li % nslot;
        const uint32_t use = li / nslot;
        if (!mbar_wait(&slot_empty[s], (use & 1) ^ 1, s_abort)) break;
        const int j = li >> 1;
        const bool hist = j < n_hist;
        const int tile = hist ? (dense ? j : tiles[j]) : j - n_hist;
        const CUtensorMap *map = (li & 1) ? (hist ? &tmV : &tmVc) : (hist ? &tmK : &tmKc);
        uint8_t *dst = ring + s * kTileBytes;
        mbar_arrive_expect_tx(&slot_full[s], kTileBytes);
        tma_load_3d(dst, map, &slot_full[s], 0, tile * BN, h);
        tma_load_3d(dst + kHalfBytes, map, &slot_full[s], 64, tile * BN, h);
        issued = li + 1;
      }
      if (*s_abort) {
        // let the copies already in flight land before the CTA goes away
        // (each wait is bounded by the same time limit)
        volatile int never = 0;
        mbar_wait(q_full, 0, &never);
        for (int li = issued - nslot < 0 ? 0 : issued - nslot; li < issued; ++li) {
          never = 0;
          mbar_wait(&slot_full[li % nslot], (li / nslot) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
      const uint32_t qa = smem_u32(sQ), ra = smem_u32(ring);
      auto issue_s = [&](int j) -> bool {
        const int li = 2 * j, s = li % nslot;
        if (!mbar_wait(&slot_full[s], (li / nslot) & 1, s_abort)) return false;
        tc_fence_after();
        const uint32_t ka = ra + s * kTileBytes;
        const uint32_t sb = tmem + (j & 1) * BN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(sb, kmajor_desc(qa, k), kmajor_desc(ka, k), idS, k > 0);
        tc_commit(&s_full[j & 1]);
        tc_commit(&slot_empty[s]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, s_abort);
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n; ++j) {
        const int b = j & 1;  // chain
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&p_full[b], ph, s_abort)) break;
        const int li = 2 * j + 1, s = li % nslot;
        if (!mbar_wait(&slot_full[s], (li / nslot) & 1, s_abort)) break;
        tc_fence_after();
        const uint32_t va = ra + s * kTileBytes;
        const uint32_t pb = tmem + b * BN;  // P_j: first 64 columns of its S buffer
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          mma_bf16_ts(tmem + kColO + b * D, pb + k * 8, vmn_desc(va, k), idPV, (j >= 2 || k > 0));
        tc_commit(&pv_done[b]);
        tc_commit(&slot_empty[s]);
        if (j + 2 < n) {
          // S_{j+2} goes into the buffer P_j occupies: PV_j must be done
          if (!mbar_wait(&pv_done[b], ph, s_abort)) break;
          if (!issue_s(j + 2)) break;
        }
      }
      // all issued MMAs must be complete before TMEM is released
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never);
    }
  } else {
    // ================= softmax / epilogue (warps 2..9) =================
    const int quarter = warp & 3;
    const int ch = (warp - 2) >> 2;     // chain: tiles j with j % 2 == ch
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t sb = trow + ch * BN;                 // this chain's S buffer
    const uint32_t ob = trow + kColO + ch * D;          // this chain's O
    const float c = a.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    int last = -1;  // this chain's last tile
    for (int j = ch; j < n; j += 2) {
      const uint32_t ph = (j >> 1) & 1;
      if (!warp_wait(&s_full[ch], ph, s_abort)) { ok = false; break; }
      tc_fence_after();
      // two passes over the S row (the register file holds 168 per thread):
      // the max, then the exponentials 32 columns at a time
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sv[64];
        tmem_ld32(sb + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(sb + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k)
          mx[k & 7] = fmax3(mx[k & 7], __uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1]));
      }
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7]));
      const float m_cand = fmaxf(m_run, mt * c);
      const bool grow = m_cand > m_run + kRescaleThreshold;  // always on the chain's first tile
      const float m_use = grow ? m_cand : m_run;
      const float alpha = fast_exp2(m_run - m_use);  // 1 if kept, 0 on the first tile
      if (last >= 0 && __any_sync(0xffffffffu, grow)) {
        // move this chain's O to the new max: its previous PV must be done
        if (!warp_wait(&pv_done[ch], (last >> 1) & 1, s_abort)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld32(ob + cc * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
          tmem_st32(ob + cc * 32, ov);
        }
      }
      // exponentials (arguments and row sum in packed pairs); P_j into the
      // first 64 columns of its S buffer: column t/2 holds elements t, t+1
      uint64_t sum2[2] = {0ull, 0ull};
      const uint64_t c2 = f2pack(c, c), nm2 = f2pack(-m_use, -m_use);
#pragma unroll
      for (int qt = 0; qt < 4; ++qt) {  // S columns 32qt.. -> P columns 16qt.. (already read)
        uint32_t sv[32];
        tmem_ld32(sb + qt * 32, sv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint64_t x2 = ffma2(f2pack(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])),
                                    c2, nm2);
          float x0, x1;
          f2unpack(x2, x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          sum2[k & 1] = fadd2(sum2[k & 1], f2pack(p0, p1));
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st16(sb + qt * 16, pk);
      }
      float sa, sb2;
      f2unpack(fadd2(sum2[0], sum2[1]), sa, sb2);
      tmem_wait_st();
      l = l * alpha + (sa + sb2);
      m_run = m_use;
      last = j;
      tc_fence_before();
      mbar_arrive(&p_full[ch]);
    }
    // epilogue: merge the two chains.  Both chains' last PVs must be done
    // before either O is read; (max, sum) per row go through shared memory
    // (the ring, idle once every PV is done).
    bool have = ok && n > 0;
    if (have) {
      for (int cc = 0; cc < 2 && cc < n; ++cc) {
        const int lc = ((n - 1) & 1) == cc ? n - 1 : n - 2;  // chain cc's last tile
        if (!mbar_wait(&pv_done[cc], (lc >> 1) & 1, s_abort)) { have = false; break; }
      }
    }
    float *xm = reinterpret_cast<float *>(ring);  // [chain][2][128]: max, sum
    xm[(ch * 2 + 0) * BM + r] = m_run;
    xm[(ch * 2 + 1) * BM + r] = l;
    mbar_arrive(x_fin);
    const bool fin_ok = mbar_wait(x_fin, 0, s_abort);
    const float mo = xm[((ch ^ 1) * 2 + 0) * BM + r];
    const float lo = xm[((ch ^ 1) * 2 + 1) * BM + r];
    const float m0 = ch == 0 ? m_run : mo, m1 = ch == 0 ? mo : m_run;
    const float l0 = ch == 0 ? l : lo, l1 = ch == 0 ? lo : l;
    const float mm = fmaxf(m0, m1);
    // a chain without tiles has max -inf and sum 0: weight 0, O never read
    const float w0 = n > 0 ? fast_exp2(m0 - mm) : 0.f;
    const float w1 = n > 1 ? fast_exp2(m1 - mm) : 0.f;
    const float l_row = l0 * w0 + l1 * w1;
    // tcgen05.ld is warp-collective: decide once for the whole warp
    const bool good = __all_sync(0xffffffffu, have && fin_ok && !*s_abort);
    tc_fence_after();
    const float inv = good ? 1.0f / l_row : 0.f;
    uint16_t *orow = a.O + ((size_t)row * BM + r) * D + ch * 64;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t o0[16], o1[16];
      if (good) {
        tmem_ld16(trow + kColO + ch * 64 + cc * 16, o0);
        if (n > 1) tmem_ld16(trow + kColO + D + ch * 64 + cc * 16, o1);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) o0[k] = 0u;
      }
      if (!good || n < 2) {
#pragma unroll
        for (int k = 0; k < 16; ++k) o1[k] = 0u;
      }
      const float s0 = w0 * inv, s1 = w1 * inv;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          v[e] = __uint_as_float(o0[8 * q + e]) * s0 + __uint_as_float(o1[8 * q + e]) * s1;
        uint4 u;
        u.x = pack_bf16x2(v[0], v[1]);
        u.y = pack_bf16x2(v[2], v[3]);
        u.z = pack_bf16x2(v[4], v[5]);
        u.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4 *>(orow + cc * 16 + q * 8) = u;
      }
    }
    if (a.lse && ch == 0)
      a.lse[(size_t)row * BM + r] = good ? (mm + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
  }

  if (*s_abort && threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_WAIT_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [H][rows][128] bf16 as a 3-D map (channel, token, head), 64 x 128 boxes.
bool make_map(CUtensorMap *map, const void *ptr, int rows, int H) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int attn_max_route() { return kMaxRoute; }

cudaError_t launch_attn(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *route_ids, const int32_t *route_len,
                        const int32_t *row_order, int R_max, const uint16_t *K_cur,
                        const uint16_t *V_cur, int N_cur, int H, int N, int M,
                        float softmax_scale, uint16_t *O, float *lse, int32_t *dev_status,
                        cudaStream_t stream, bool *map_failed) {
  *map_failed = false;
  CUtensorMap mq, mk, mv, mkc, mvc;
  const bool cur = K_cur != nullptr && N_cur > 0;
  if (!make_map(&mq, Q, N * BM, H) || !make_map(&mk, K, M * BN, H) ||
      !make_map(&mv, V, M * BN, H) ||
      !make_map(&mkc, cur ? K_cur : K, cur ? N_cur * BN : M * BN, H) ||
      !make_map(&mvc, cur ? V_cur : V, cur ? N_cur * BN : M * BN, H)) {
    *map_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnArgs a;
  a.Q = Q;
  a.route_ids = route_ids;
  a.route_len = route_len;
  a.row_order = row_order;
  a.R_max = R_max;
  a.N = N;
  a.M = M;
  a.rows = H * N;
  a.n_cur = cur ? N_cur : 0;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.O = O;
  a.lse = lse;
  a.dev_status = dev_status;
  // tail after the ring: barriers, misc, route list (uint16), id bitmap
  const uint32_t list_bytes = route_ids ? ((uint32_t)R_max * 2u + 15u) & ~15u : 0u;
  const uint32_t bits_bytes = route_ids ? (uint32_t)((M + 31) / 32) * 4u : 0u;
  const uint32_t tail = kNumBars * 8 + kMiscBytes + list_bytes + bits_bytes;
  int nslot = kMaxSlots;
  while (nslot > 4 && kOffRing + nslot * kTileBytes + tail + 1024 > kSmemLimit) --nslot;
  // loads go K_0, V_0, K_1, V_1, ... round the ring; load li reuses the slot
  // of load li - nslot.  With an odd count K_{j+3} would reuse V_j's slot and
  // could not start before PV_j, just when S_{j+3} is wanted: keep it even.
  nslot &= ~1;
  a.nslot = nslot;
  a.bar_offset = kOffRing + nslot * kTileBytes;
  a.list_offset = a.bar_offset + kNumBars * 8 + kMiscBytes;
  a.bits_offset = a.list_offset + list_bytes;
  const size_t smem = (size_t)a.bits_offset + bits_bytes + 1024;  // + alignment slack
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  attn_kernel<<<H * N, kThreads, smem, stream>>>(mq, mk, mv, mkc, mvc, a);
  return cudaGetLastError();
}

}  // namespace velox
