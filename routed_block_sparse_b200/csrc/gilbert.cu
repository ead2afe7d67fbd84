// Global-aligned Gilbert order and 26-neighbour safeguard blocks.
//
// Velox project page, "02 · Method", "Keeping neighbours adjacent in the
// block order" and figure "Incremental Gilbert order": the KV cache is stored
// in a Gilbert space-filling order, built once per frame and mirrored on
// alternate frames so that frame and chunk seams stay adjacent; 128-token
// blocks of that order are the route ids, and lattice neighbours of a query
// block are safeguards (digest of arXiv 2610.22311, "Method steps", Eq. 14).
//
// Instead of generating the curve sequentially, every thread locates its own
// cell by descending the generalised-Hilbert recursion: at each level the
// rectangle is cut into two (long rectangles) or three pieces, the piece
// holding the cell is found by a containment test, and the sizes of the
// pieces walked before it are added to the rank.  The depth is O(log(WH)).
// The inverse (rank -> cell) descends the same recursion by piece sizes.
#include "common.cuh"

namespace velox {
namespace {

struct Rect {
  int x, y;    // start corner
  int ax, ay;  // major edge vector
  int bx, by;  // minor edge vector
};

__device__ __forceinline__ int sgn(int v) { return (v > 0) - (v < 0); }
// floor(v / 2) for negative v as well (the recursion halves signed vectors)
__device__ __forceinline__ int floor_half(int v) { return (v - (v & 1)) / 2; }
__device__ __forceinline__ int iabs(int v) { return v < 0 ? -v : v; }

__device__ __forceinline__ bool contains(const Rect &r, int cx, int cy) {
  int ux = sgn(r.ax), uy = sgn(r.ay), vx = sgn(r.bx), vy = sgn(r.by);
  int i = (cx - r.x) * ux + (cy - r.y) * uy;
  int j = (cx - r.x) * vx + (cy - r.y) * vy;
  return i >= 0 && i < iabs(r.ax + r.ay) && j >= 0 && j < iabs(r.bx + r.by);
}

__device__ __forceinline__ int area(const Rect &r) {
  return iabs(r.ax + r.ay) * iabs(r.bx + r.by);
}

// One recursion level: a rectangle is cut across its major edge into two
// halves (long rectangles) or into three pieces (the near half of the minor
// edge with the edges swapped, the full-length remainder, and a mirrored piece
// returning along the far side); halves are made even when the edge is longer
// than 2.  piece(r, q) builds piece q of r; pieces(r) is their number, 0 for a
// one-cell-thick rectangle (a straight line).  No arrays: the descent keeps
// everything in registers.
__device__ __forceinline__ int pieces(const Rect &r) {
  const int nmaj = iabs(r.ax + r.ay), nmin = iabs(r.bx + r.by);
  if (nmin == 1 || nmaj == 1) return 0;
  return 2 * nmaj > 3 * nmin ? 2 : 3;
}
__device__ __forceinline__ Rect piece(const Rect &r, int q) {
  const int nmaj = iabs(r.ax + r.ay), nmin = iabs(r.bx + r.by);
  const int ux = sgn(r.ax), uy = sgn(r.ay), vx = sgn(r.bx), vy = sgn(r.by);
  int hax = floor_half(r.ax), hay = floor_half(r.ay);
  int hbx = floor_half(r.bx), hby = floor_half(r.by);
  if (2 * nmaj > 3 * nmin) {
    if ((iabs(hax + hay) & 1) && nmaj > 2) { hax += ux; hay += uy; }
    if (q == 0) return {r.x, r.y, hax, hay, r.bx, r.by};
    return {r.x + hax, r.y + hay, r.ax - hax, r.ay - hay, r.bx, r.by};
  }
  if ((iabs(hbx + hby) & 1) && nmin > 2) { hbx += vx; hby += vy; }
  if (q == 0) return {r.x, r.y, hbx, hby, hax, hay};
  if (q == 1) return {r.x + hbx, r.y + hby, r.ax, r.ay, r.bx - hbx, r.by - hby};
  return {r.x + (r.ax - ux) + (hbx - vx), r.y + (r.ay - uy) + (hby - vy), -hbx, -hby,
          -(r.ax - hax), -(r.ay - hay)};
}

// Position of cell (cx, cy) on the curve of a W x H frame (W >= H).
__device__ int frame_rank(int W, int H, int cx, int cy) {
  Rect r = {0, 0, W, 0, 0, H};
  int base = 0;
  for (;;) {
    const int n = pieces(r);
    if (n == 0) {
      // a line: along the major edge if it is one cell thick, else the minor
      if (iabs(r.bx + r.by) == 1)
        return base + (cx - r.x) * sgn(r.ax) + (cy - r.y) * sgn(r.ay);
      return base + (cx - r.x) * sgn(r.bx) + (cy - r.y) * sgn(r.by);
    }
    Rect p = piece(r, 0);
    int q = 0;
    while (q < n - 1 && !contains(p, cx, cy)) {
      base += area(p);
      p = piece(r, ++q);
    }
    r = p;
  }
}

// Cell at position k of the curve of a W x H frame.
__device__ void frame_cell(int W, int H, int k, int &cx, int &cy) {
  Rect r = {0, 0, W, 0, 0, H};
  for (;;) {
    const int n = pieces(r);
    if (n == 0) {
      if (iabs(r.bx + r.by) == 1) {
        cx = r.x + k * sgn(r.ax);
        cy = r.y + k * sgn(r.ay);
      } else {
        cx = r.x + k * sgn(r.bx);
        cy = r.y + k * sgn(r.by);
      }
      return;
    }
    Rect p = piece(r, 0);
    int q = 0;
    while (q < n - 1 && k >= area(p)) {
      k -= area(p);
      p = piece(r, ++q);
    }
    r = p;
  }
}

struct Lattice {
  int T, H, W, n_chunks, b;
  int thw;  // 1: THW-linear (raster) order instead of the global Gilbert order
  __device__ int HW() const { return H * W; }
  __device__ bool mirrored(int f) const { return !thw && (f & 1); }
  // position of in-frame cell (x, y) on the frame's walk
  __device__ int in_frame(int x, int y) const { return thw ? y * W + x : frame_rank(W, H, x, y); }
  // global rank of cell (f, y, x)
  __device__ int rank(int f, int y, int x) const {
    int xm = mirrored(f) ? (W - 1 - x) : x;
    return f * H * W + in_frame(xm, y);
  }
};

__global__ void order_kernel(Lattice L, int n_cells, int32_t *rank_of_cell,
                             int32_t *cell_of_rank, int32_t *block_of_cell) {
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < n_cells; c += gridDim.x * blockDim.x) {
    int f = c / L.HW();
    int rem = c - f * L.HW();
    int y = rem / L.W;
    int x = rem - y * L.W;
    int r = L.rank(f, y, x);
    if (rank_of_cell) rank_of_cell[c] = r;
    if (cell_of_rank) cell_of_rank[r] = c;
    if (block_of_cell) block_of_cell[c] = r / L.b;
  }
}

// One CTA per query block i of chunk q_chunk.  The neighbours of a block
// whose tokens span global frames f0..f1 lie in frames f0-1 .. f1+1, hence in
// a window of block ids [wlo, whi]; a bitmap over that window collects them
// without repeats, and a scan of the bitmap writes them in ascending order.
// When a frame has at most kFrameSmemCells cells, the frame's rank map and its
// inverse are built once in shared memory and every lookup is a table read;
// otherwise each lookup descends the recursion.
constexpr int kFrameSmemCells = 8192;
constexpr int kNbrThreads = 512;

__global__ void neighbour_kernel(Lattice L, int q_chunk, int cache_first, int n_cache,
                                 int32_t *nbr_ids, int32_t *nbr_cnt, int S_max, int use_table,
                                 int32_t *dev_status) {
  extern __shared__ int smem_i[];
  __shared__ int s_scan[kNbrThreads];
  const int HW = L.HW();
  int *r2 = smem_i;                             // [HW] when use_table
  int *inv = smem_i + (use_table ? HW : 0);     // [HW] when use_table
  uint32_t *win = reinterpret_cast<uint32_t *>(smem_i + (use_table ? 2 * HW : 0));
  const int per_chunk = L.T * HW / L.b;
  const int i = blockIdx.x;
  const int qb = q_chunk * per_chunk + i;
  const int F = L.n_chunks * L.T;
  const long long first_rank = (long long)qb * L.b;
  const int f0 = (int)(first_rank / HW), f1 = (int)((first_rank + L.b - 1) / HW);
  const int wf0 = f0 > 0 ? f0 - 1 : 0, wf1 = f1 + 1 < F ? f1 + 1 : F - 1;
  const int wlo = (int)((long long)wf0 * HW / L.b);
  const int whi = (int)(((long long)(wf1 + 1) * HW - 1) / L.b);
  const int nwin = whi - wlo + 1;
  const int nwords = (nwin + 31) >> 5;
  for (int k = threadIdx.x; k < nwords; k += blockDim.x) win[k] = 0u;
  if (use_table) {
    for (int cidx = threadIdx.x; cidx < HW; cidx += blockDim.x) {
      const int y = cidx / L.W, x = cidx - y * L.W;
      const int rk = L.in_frame(x, y);
      r2[cidx] = rk;
      inv[rk] = cidx;
    }
  }
  __syncthreads();
  const int items = L.b * 26;
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int t = it / 26, o26 = it - t * 26;
    const int o = o26 < 13 ? o26 : o26 + 1;  // skip the centre offset 13
    const long long rank = first_rank + t;
    const int f = (int)(rank / HW);
    const int k = (int)(rank - (long long)f * HW);
    int xm, y;
    if (use_table) {
      const int cidx = inv[k];
      y = cidx / L.W;
      xm = cidx - y * L.W;
    } else if (L.thw) {
      y = k / L.W;
      xm = k - y * L.W;
    } else {
      frame_cell(L.W, L.H, k, xm, y);
    }
    const int x = L.mirrored(f) ? (L.W - 1 - xm) : xm;
    const int f2 = f + o / 9 - 1, y2 = y + (o / 3) % 3 - 1, x2 = x + o % 3 - 1;
    if (f2 < 0 || f2 >= F || y2 < 0 || y2 >= L.H || x2 < 0 || x2 >= L.W) continue;
    const int xm2 = L.mirrored(f2) ? (L.W - 1 - x2) : x2;
    const int r2v = use_table ? r2[y2 * L.W + xm2] : L.in_frame(xm2, y2);
    const int u = (int)(((long long)f2 * HW + r2v) / L.b);
    if (u == qb || u < cache_first || u >= cache_first + n_cache) continue;
    const int bit = u - wlo;  // within the window by construction
    atomicOr(&win[bit >> 5], 1u << (bit & 31));
  }
  __syncthreads();
  // ordered write-out: thread t owns a contiguous run of bitmap words
  const int wchunk = (nwords + blockDim.x - 1) / blockDim.x;
  const int wl = min(nwords, (int)threadIdx.x * wchunk), wh = min(nwords, wl + wchunk);
  int mine = 0;
  for (int k = wl; k < wh; ++k) mine += __popc(win[k]);
  s_scan[threadIdx.x] = mine;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    int v = threadIdx.x >= (unsigned)off ? s_scan[threadIdx.x - off] : 0;
    __syncthreads();
    s_scan[threadIdx.x] += v;
    __syncthreads();
  }
  const int total = s_scan[blockDim.x - 1];
  int pos = s_scan[threadIdx.x] - mine;
  for (int k = wl; k < wh; ++k) {
    uint32_t w = win[k];
    while (w) {
      const int bit = __ffs(w) - 1;
      w &= w - 1;
      if (pos < S_max && nbr_ids) nbr_ids[(size_t)i * S_max + pos] = wlo + (k << 5) + bit - cache_first;
      ++pos;
    }
  }
  for (int k = total + threadIdx.x; k < S_max; k += blockDim.x)
    if (nbr_ids) nbr_ids[(size_t)i * S_max + k] = -1;
  if (threadIdx.x == 0) {
    if (nbr_cnt) nbr_cnt[i] = min(total, S_max);
    if (total > S_max) flag_error(dev_status, VELOX_DEV_NBR_OVERFLOW);
  }
}

}  // namespace

cudaError_t launch_gilbert(int T, int H, int W, int n_chunks, int b, int q_chunk,
                           int cache_first, int n_cache, int32_t *rank_of_cell,
                           int32_t *cell_of_rank, int32_t *block_of_cell, int32_t *nbr_ids,
                           int32_t *nbr_cnt, int S_max, int thw, int32_t *dev_status,
                           cudaStream_t stream) {
  Lattice L{T, H, W, n_chunks, b, thw};
  const int n_cells = n_chunks * T * H * W;
  if (rank_of_cell || cell_of_rank || block_of_cell) {
    int grid = (n_cells + 255) / 256;
    if (grid > 148 * 32) grid = 148 * 32;
    order_kernel<<<grid, 256, 0, stream>>>(L, n_cells, rank_of_cell, cell_of_rank,
                                           block_of_cell);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (nbr_ids || nbr_cnt) {
    const int HW = H * W;
    const int per_chunk = T * HW / b;
    const int use_table = HW <= kFrameSmemCells ? 1 : 0;
    // window of candidate block ids: at most (frames spanned + 2) frames
    const long long span_frames = (b + HW - 1) / HW + 1;
    const long long nwin = ((span_frames + 2) * HW) / b + 2;
    size_t smem = (use_table ? (size_t)2 * HW * sizeof(int) : 0) +
                  (size_t)((nwin + 31) / 32) * sizeof(uint32_t);
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(neighbour_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    neighbour_kernel<<<per_chunk, kNbrThreads, smem, stream>>>(L, q_chunk, cache_first, n_cache,
                                                       nbr_ids, nbr_cnt, S_max, use_table,
                                                       dev_status);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace velox
