// Soft geometry fusion and route materialisation.
//
// Velox project page, "02 · Method": p~_{i,r} ~ p_{i,r} (1 + lambda g^_{i,r}),
// g^ = [g > tau] min(g / g_ref, 1), for covered query blocks; uncovered blocks
// keep the model's own p ("Covered and uncovered blocks").  Digest of arXiv
// 2610.22311, "Method steps", Eq. 12-14, and onedev.kr summary, "How it
// differs": sort descending, take the minimal cumulative-mass prefix capped at
// K_cov / K_unc, previous chunk reserved inside the budget, 26-neighbour and
// reference blocks appended outside it.
//
// One CTA per (head, query block) row:
//   1. fused weights w_r in fp64 (explicit round-to-nearest operations, so
//      no contraction changes the value), row sum Z;
//   2. radix select (passes of 8 bits over an order-preserving 64-bit key,
//      from the highest byte in which the eligible keys differ) of the k
//      largest non-reserved weights, ties to the lower id;
//   3. rank sort of the <= k survivors (weight desc, id asc);
//   4. warp scan of the normalised mass from the reserved mass on: the cut is
//      the first position at which the mass before it reaches theta;
//   5. budget / safeguard bitmaps, written out in ascending id order.
#include "common.cuh"

namespace velox {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// up to this many candidates are ordered by a rank sort (O(k^2 / threads)
// compares); more by a bitonic network in shared memory (O(k log^2 k))
constexpr int kRankSortMax = 256;

struct RouteArgs {
  const float *p;
  const float *g;
  const uint8_t *covered;
  double lam, tau, g_ref, theta_cov, theta_unc;
  int k_cov, k_unc;
  int prev_begin, prev_count;
  const int32_t *nbr_ids;
  const int32_t *nbr_cnt;
  int S_max;
  const int32_t *ref_ids;
  int n_ref;
  int N, M;
  int32_t *route_ids, *route_len, *route_nbudget;
  int R_max;
  double *ws_keys;  // [rows][M] when the keys do not fit in shared memory
  int kcap;         // candidate capacity = max(k_cov, k_unc) (>= 1), rounded up to a
                    // power of two when above kRankSortMax (the bitonic sort's length)
  int32_t *dev_status;
};

// Order-preserving map of a double onto uint64 (larger double -> larger key).
__device__ __forceinline__ uint64_t order_key(double w) {
  uint64_t b = static_cast<uint64_t>(__double_as_longlong(w));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ double block_sum(double v, double *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kWarps; ++w) t += scratch[w];  // fixed order
  return t;
}

// Exclusive scan of one int per thread over the block; *total gets the sum.
__device__ int block_excl_scan(int v, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before += scratch[w];
    all += scratch[w];
  }
  *total = all;
  return before + incl - v;
}

// six rows per SM: the register cap (40) costs a few bytes of spills and
// keeps 2.2 waves at the chunk-48 shape instead of 3.2
__global__ void __launch_bounds__(kThreads, 6) route_kernel(RouteArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ double s_dred[kWarps];
  __shared__ int s_ired[kWarps];
  __shared__ int s_hist[256];
  __shared__ int s_digit, s_greater, s_equal, s_ntake;
  __shared__ uint64_t s_kand[kWarps], s_kor[kWarps];

  const int row = blockIdx.x;
  const int i = row % a.N;
  const int M = a.M;
  const int tid = threadIdx.x;
  const int W = (M + 31) >> 5;

  // ---- shared-memory carve-up
  unsigned char *cur = smem_raw;
  double *cand_key = reinterpret_cast<double *>(cur); cur += sizeof(double) * a.kcap;
  double *sort_s = reinterpret_cast<double *>(cur); cur += sizeof(double) * a.kcap;
  int *cand_id = reinterpret_cast<int *>(cur); cur += sizeof(int) * a.kcap;
  int *sort_id = reinterpret_cast<int *>(cur); cur += sizeof(int) * a.kcap;
  uint32_t *bud_bits = reinterpret_cast<uint32_t *>(cur); cur += sizeof(uint32_t) * W;
  uint32_t *ext_bits = reinterpret_cast<uint32_t *>(cur); cur += sizeof(uint32_t) * W;
  cur = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(cur) + 15) & ~uintptr_t(15));
  double *keys = a.ws_keys ? a.ws_keys + (size_t)row * M : reinterpret_cast<double *>(cur);

  const bool cov = a.covered[i] != 0;
  const int K = cov ? a.k_cov : a.k_unc;
  const double theta = cov ? a.theta_cov : a.theta_unc;
  const int pb = a.prev_begin, pe = a.prev_begin + a.prev_count;
  const float *prow = a.p + (size_t)row * M;
  const float *grow = a.g + (size_t)i * M;

  for (int k = tid; k < W; k += kThreads) { bud_bits[k] = 0u; ext_bits[k] = 0u; }

  // ---- 1. fused weights and their sum
  // loads four deep per thread (the same ids and summation order as a plain
  // strided loop): one memory round trip per four keys
  double zpart = 0.0;
  constexpr int kBatch = 4;
  for (int base = tid; base < M; base += kThreads * kBatch) {
    float pf[kBatch], gf[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = base + u * kThreads;
      pf[u] = r < M ? __ldg(prow + r) : 0.f;
      gf[u] = (cov && r < M) ? __ldg(grow + r) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = base + u * kThreads;
      if (r >= M) break;
      const double pv = static_cast<double>(pf[u]);
      double w = pv;
      if (cov) {
        const double gv = static_cast<double>(gf[u]);
        double gh = 0.0;
        if (gv > a.tau) {
          gh = __ddiv_rn(gv, a.g_ref);
          if (gh > 1.0) gh = 1.0;
        }
        w = __dmul_rn(pv, __dadd_rn(1.0, __dmul_rn(a.lam, gh)));
      }
      w = __dadd_rn(w, 0.0);  // -0 -> +0, so that zeros tie exactly
      keys[r] = w;
      zpart += w;
    }
  }
  const double Z = cov ? block_sum(zpart, s_dred) : 1.0;
  const double invZ_ok = (Z > 0.0) ? 1.0 : 0.0;  // Z == 0: no mass ever counts
  __syncthreads();

  // ---- reserved mass
  double mpart = 0.0;
  for (int r = pb + tid; r < pe; r += kThreads)
    mpart += cov ? (invZ_ok != 0.0 ? __ddiv_rn(keys[r], Z) : 0.0) : keys[r];
  const double mass_P = block_sum(mpart, s_dred);

  const int n_res = a.prev_count;
  const int n_elig = M - n_res;
  int k_sel = K - n_res;
  if (k_sel > n_elig) k_sel = n_elig;
  if (k_sel < 0 || !(mass_P < theta)) k_sel = 0;

  // ---- 2. radix select of the k_sel-th largest eligible key
  uint64_t prefix = 0, mask = 0;
  int need = k_sel;
  const bool select_all = (k_sel == n_elig);
  if (k_sel > 0 && !select_all) {
    // bytes that every eligible key shares decide nothing: start below them
    uint64_t kand = ~0ull, kor = 0ull;
    for (int r = tid; r < M; r += kThreads) {
      if (r >= pb && r < pe) continue;
      const uint64_t u = order_key(keys[r]);
      kand &= u;
      kor |= u;
    }
    const uint32_t a_hi = __reduce_and_sync(0xffffffffu, (uint32_t)(kand >> 32));
    const uint32_t a_lo = __reduce_and_sync(0xffffffffu, (uint32_t)kand);
    const uint32_t o_hi = __reduce_or_sync(0xffffffffu, (uint32_t)(kor >> 32));
    const uint32_t o_lo = __reduce_or_sync(0xffffffffu, (uint32_t)kor);
    if ((tid & 31) == 0) {
      s_kand[tid >> 5] = ((uint64_t)a_hi << 32) | a_lo;
      s_kor[tid >> 5] = ((uint64_t)o_hi << 32) | o_lo;
    }
    __syncthreads();
    uint64_t all_and = ~0ull, all_or = 0ull;
    for (int w = 0; w < kWarps; ++w) {
      all_and &= s_kand[w];
      all_or |= s_kor[w];
    }
    const uint64_t diff = all_and ^ all_or;
    int shift0;
    if (diff == 0ull) {
      shift0 = -8;  // every eligible key is equal: all of them tie
      mask = ~0ull;
      prefix = all_and;
    } else {
      const int hb = 63 - __clzll(static_cast<long long>(diff));
      shift0 = (hb >> 3) << 3;
      mask = (shift0 >= 56) ? 0ull : ~((1ull << (shift0 + 8)) - 1ull);
      prefix = all_and & mask;
    }
    for (int shift = shift0; shift >= 0; shift -= 8) {
      for (int k = tid; k < 256; k += kThreads) s_hist[k] = 0;
      __syncthreads();
      // warp-aggregated: keys mostly share their leading digits, so one
      // atomic per distinct digit per warp instead of one per key
      for (int base = 0; base < M; base += kThreads) {
        const int r = base + tid;
        int digit = -1;
        if (r < M && !(r >= pb && r < pe)) {
          const uint64_t u = order_key(keys[r]);
          if ((u & mask) == prefix) digit = static_cast<int>((u >> shift) & 255u);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, digit);
        if (digit >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&s_hist[digit], __popc(peers));
      }
      __syncthreads();
      if (tid < 32) {
        // lane l holds digits 255-8l .. 248-8l (descending)
        int c[8], lt = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { c[j] = s_hist[255 - 8 * tid - j]; lt += c[j]; }
        int incl = lt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          int o = __shfl_up_sync(0xffffffffu, incl, off);
          if (tid >= off) incl += o;
        }
        int run = incl - lt;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < need && run + c[j] >= need) {
            s_digit = 255 - 8 * tid - j;
            s_greater = run;
            s_equal = c[j];
          }
          run += c[j];
        }
      }
      __syncthreads();
      prefix |= static_cast<uint64_t>(s_digit) << shift;
      mask |= 0xFFull << shift;
      need -= s_greater;
      const bool all_of_digit = (need == s_equal);
      __syncthreads();
      // every key that shares the prefix so far is taken: the lower bytes
      // cannot change the selection
      if (all_of_digit) break;
    }
  }
  // keys are compared on their bytes under `mask`: prefix = those bytes of
  // the k_sel-th largest; `need` keys equal to it there are taken, lowest
  // ids first.

  // ---- compaction in id order (thread t owns ids [t*c, t*c + c))
  const int chunk = (M + kThreads - 1) / kThreads;
  const int lo = min(M, tid * chunk), hi = min(M, lo + chunk);
  int n_gt = 0, n_tie = 0;
  if (k_sel > 0) {
    for (int r = lo; r < hi; ++r) {
      if (r >= pb && r < pe) continue;
      if (select_all) { ++n_gt; continue; }
      const uint64_t u = order_key(keys[r]) & mask;
      n_gt += (u > prefix);
      n_tie += (u == prefix);
    }
  }
  int tot;
  const int tie_before = block_excl_scan(n_tie, s_ired, &tot);
  int take_tie = need - tie_before;
  take_tie = take_tie < 0 ? 0 : (take_tie > n_tie ? n_tie : take_tie);
  if (select_all) take_tie = 0;
  const int pos0 = block_excl_scan(n_gt + take_tie, s_ired, &tot);
  if (k_sel > 0) {
    int pos = pos0, ties_seen = 0;
    for (int r = lo; r < hi; ++r) {
      if (r >= pb && r < pe) continue;
      bool inc;
      if (select_all) {
        inc = true;
      } else {
        const uint64_t u = order_key(keys[r]) & mask;
        inc = (u > prefix) || (u == prefix && ties_seen++ < take_tie);
      }
      if (inc && pos < a.kcap) {
        cand_id[pos] = r;
        cand_key[pos] = keys[r];
        ++pos;
      }
    }
  }
  __syncthreads();

  // ---- 3. sort the candidates: weight descending, ties to the lower id
  //         (candidates arrive in id order)
  if (k_sel <= kRankSortMax) {
    for (int x = tid; x < k_sel; x += kThreads) {
      const double kx = cand_key[x];
      int rank = 0;
      for (int y = 0; y < k_sel; ++y) {
        const double ky = cand_key[y];
        rank += (ky > kx) || (ky == kx && y < x);
      }
      sort_id[rank] = cand_id[x];
      sort_s[rank] = cov ? (invZ_ok != 0.0 ? __ddiv_rn(kx, Z) : 0.0) : kx;
    }
  } else {
    // bitonic network over the next power of two; padding (-1, INT_MAX)
    // sorts after every weight (weights are >= 0)
    int P = 1;
    while (P < k_sel) P <<= 1;
    for (int x = k_sel + tid; x < P; x += kThreads) {
      cand_key[x] = -1.0;
      cand_id[x] = 0x7FFFFFFF;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int x = tid; x < P; x += kThreads) {
          const int y = x ^ jj;
          if (y > x) {
            const double kx = cand_key[x], ky = cand_key[y];
            const int ix = cand_id[x], iy = cand_id[y];
            const bool x_first = (kx > ky) || (kx == ky && ix < iy);
            // segments with (x & k) == 0 end up in the output order
            if (((x & k) == 0) != x_first) {
              cand_key[x] = ky; cand_key[y] = kx;
              cand_id[x] = iy; cand_id[y] = ix;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int q = tid; q < k_sel; q += kThreads) {
      const double kq = cand_key[q];
      sort_id[q] = cand_id[q];
      sort_s[q] = cov ? (invZ_ok != 0.0 ? __ddiv_rn(kq, Z) : 0.0) : kq;
    }
  }
  __syncthreads();

  // ---- 4. the cut: first position whose preceding mass reaches theta
  if (tid < 32) {
    double run = mass_P;
    int cut = k_sel;
    for (int base = 0; base < k_sel; base += 32) {
      const int q = base + tid;
      const double v = q < k_sel ? sort_s[q] : 0.0;
      double incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        double o = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += o;
      }
      const double before = run + (incl - v);
      const unsigned hit = __ballot_sync(0xffffffffu, q < k_sel && before >= theta);
      if (hit) { cut = base + __ffs(hit) - 1; break; }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) s_ntake = cut;
  }
  __syncthreads();
  const int n_take = s_ntake;

  // ---- 5. budget bitmap, safeguards, ordered output
  for (int r = pb + tid; r < pe; r += kThreads) atomicOr(&bud_bits[r >> 5], 1u << (r & 31));
  for (int q = tid; q < n_take; q += kThreads) {
    const int r = sort_id[q];
    atomicOr(&bud_bits[r >> 5], 1u << (r & 31));
  }
  __syncthreads();
  int ncnt = 0;
  if (a.nbr_ids && a.nbr_cnt && a.S_max > 0) {
    ncnt = a.nbr_cnt[i];
    if (ncnt < 0 || ncnt > a.S_max) {
      flag_error(a.dev_status, VELOX_DEV_BAD_SAFEGUARD);
      ncnt = ncnt < 0 ? 0 : a.S_max;
    }
  }
  for (int q = tid; q < ncnt + a.n_ref; q += kThreads) {
    const int u = q < ncnt ? a.nbr_ids[(size_t)i * a.S_max + q] : a.ref_ids[q - ncnt];
    if (u < 0 || u >= M) {
      flag_error(a.dev_status, VELOX_DEV_BAD_SAFEGUARD);
      continue;
    }
    if (!(bud_bits[u >> 5] & (1u << (u & 31)))) atomicOr(&ext_bits[u >> 5], 1u << (u & 31));
  }
  __syncthreads();

  const int wchunk = (W + kThreads - 1) / kThreads;
  const int wlo = min(W, tid * wchunk), whi = min(W, wlo + wchunk);
  int nb_mine = 0, ne_mine = 0;
  for (int k = wlo; k < whi; ++k) { nb_mine += __popc(bud_bits[k]); ne_mine += __popc(ext_bits[k]); }
  int nb, ne;
  const int bpos0 = block_excl_scan(nb_mine, s_ired, &nb);
  const int epos0 = block_excl_scan(ne_mine, s_ired, &ne);
  int32_t *out = a.route_ids + (size_t)row * a.R_max;
  if (nb + ne > a.R_max) flag_error(a.dev_status, VELOX_DEV_ROUTE_CAPACITY);
  int bp = bpos0, ep = nb + epos0;
  for (int k = wlo; k < whi; ++k) {
    uint32_t bw = bud_bits[k], ew = ext_bits[k];
    while (bw) {
      const int bit = __ffs(bw) - 1;
      bw &= bw - 1;
      if (bp < a.R_max) out[bp] = (k << 5) + bit;
      ++bp;
    }
    while (ew) {
      const int bit = __ffs(ew) - 1;
      ew &= ew - 1;
      if (ep < a.R_max) out[ep] = (k << 5) + bit;
      ++ep;
    }
  }
  for (int k = nb + ne + tid; k < a.R_max; k += kThreads) out[k] = -1;
  if (tid == 0) {
    a.route_len[row] = min(nb + ne, a.R_max);
    a.route_nbudget[row] = min(nb, a.R_max);
  }
}

}  // namespace

// Keys of a row live in shared memory up to this many history blocks, else
// in the workspace.
constexpr int kSmemKeysMaxM = 12288;

size_t route_workspace_bytes(int H, int N, int M) {
  if (M <= kSmemKeysMaxM) return 0;
  return ((size_t)H * N * M * sizeof(double) + 255) & ~(size_t)255;
}

// Candidate capacity: max(k_cov, k_unc), at least 1, rounded up to a power
// of two when the bitonic sort is used.
int route_kcap(int k_cov, int k_unc) {
  int k = k_cov > k_unc ? k_cov : k_unc;
  if (k < 1) k = 1;
  if (k > kRankSortMax) {
    int p = 1;
    while (p < k) p <<= 1;
    k = p;
  }
  return k;
}

size_t route_smem_bytes(int M, int kcap) {
  const int W = (M + 31) / 32;
  size_t b = (size_t)kcap * (8 + 8 + 4 + 4) + (size_t)W * 8;
  b = (b + 15) & ~(size_t)15;
  if (M <= kSmemKeysMaxM) b += (size_t)M * 8;
  return b;
}

cudaError_t launch_route(const float *p, const float *g, const uint8_t *covered,
                         const velox_route_params *prm, int prev_begin, int prev_count,
                         const int32_t *nbr_ids, const int32_t *nbr_cnt, int S_max,
                         const int32_t *ref_ids, int n_ref, int H, int N, int M,
                         int32_t *route_ids, int32_t *route_len, int32_t *route_nbudget,
                         int R_max, void *ws, int32_t *dev_status, cudaStream_t stream) {
  RouteArgs a;
  a.p = p; a.g = g; a.covered = covered;
  a.lam = prm->lambda; a.tau = prm->tau; a.g_ref = prm->g_ref;
  a.theta_cov = prm->theta_cov; a.theta_unc = prm->theta_unc;
  a.k_cov = prm->k_cov; a.k_unc = prm->k_unc;
  a.prev_begin = prev_begin; a.prev_count = prev_count;
  a.nbr_ids = nbr_ids; a.nbr_cnt = nbr_cnt; a.S_max = S_max;
  a.ref_ids = ref_ids; a.n_ref = n_ref;
  a.N = N; a.M = M;
  a.route_ids = route_ids; a.route_len = route_len; a.route_nbudget = route_nbudget;
  a.R_max = R_max;
  a.ws_keys = (M <= kSmemKeysMaxM) ? nullptr : static_cast<double *>(ws);
  a.kcap = route_kcap(prm->k_cov, prm->k_unc);
  a.dev_status = dev_status;
  const size_t smem = route_smem_bytes(M, a.kcap);
  cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  route_kernel<<<H * N, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace velox
