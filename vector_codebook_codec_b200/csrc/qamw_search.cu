// qamw_search.cu -- candidate table for the exact pruned nearest-centroid search.
//
// Methodology (4) Joint 2D Quantization of the QAM-W page maps each normalised
// pair x to the nearest centroid of one 2D codebook. The brute-force search
// computes N distances per pair. This table lets the encode compute only the
// distances that can matter. Each axis is mapped by the monotone
// T(x) = x / (a + |x|), and the square [-L, L]^2 (L well beyond the outermost
// centroid) is cut into G x G cells uniform in (T(x0), T(x1)): the cells are
// small near the origin, where the pairs (unit circular Gaussian after the
// sigma normalisation) and the centroids are dense, and grow outwards. For
// every cell Q (enlarged by a small margin) the table lists every centroid c
// with
//     dmin(c, Q)^2 <= (1 + 1e-5) * D(Q)^2,   D(Q) = min_c' dmax(c', Q),
// dmin / dmax being the least / greatest distance from c to a point of Q.
// For a pair x in Q its exact nearest distance d* is at most D(Q), and every
// centroid whose fp32 direct-difference distance ties or beats the fp32
// distance of the exact nearest one is within a factor (1 + 4e-7) of d*, so
// it passes this first test.
//
// The first test keeps every centroid whose disc of radius D(Q) meets Q; a
// second one drops the members that another member beats everywhere in Q.
// Member c is dropped if some member c' has
//     |p - c|^2 > (1 + 1e-5) |p - c'|^2   at the four corners p of Q.
// f(p) = |p - c|^2 - (1 + 1e-5) |p - c'|^2 is -1e-5 |p|^2 plus terms of degree
// at most one, a concave function, so its least value over the rectangle Q is
// taken at a corner: f > 0 at the corners means f > 0 on all of Q. The fp32
// distances of c and c' are within a factor (1 + 4e-7) of the exact ones, so
// at every pair in Q the fp32 distance of c is strictly greater than that of
// c': c is never the fp32 minimiser nor tied with it. (If c' is dropped in
// turn, the member that beats c' beats c too.) The fp32 minimisers of every
// pair in Q are therefore all kept, and scanning a cell's list in ascending
// index order with a strict "<" returns exactly the index of the brute-force
// search (the lowest index among the fp32 minimisers). A first-test list longer
// than kListMax is kept whole. Pairs outside the grid, or a table that does
// not fit, use the brute-force search.
//
// The encode computes a pair's cell in fp32 as round(T(x) * inv_cw + (G-1)/2),
// which for odd G is floor((T(x) + UL) * inv_cw), with inv_cw, a and L read
// from the header (search_cell in qamw_internal.h); its error is below 1e-4
// of a cell, and the margin of 1e-3 cells that every cell is enlarged by (in
// u, then mapped back to x in fp64) covers it.
//
// Table layout (device memory owned by the caller, 16-byte aligned):
//   SearchHeader (48 bytes, padded to 64) | uint64 rec[G*G] | uint16 ovf[capacity]
// rec[k] is the record of cell k = iy * G + ix (qamw_internal.h): up to three
// candidates inline, longer lists continue in ovf. The records and the
// overflow array form one image of image_bytes that the encode copies to
// shared memory with one bulk asynchronous copy. Short lists (one to three
// entries, ~96% of the pairs on the shipped N = 2048 codebook at G = 137)
// need no list load at all: the record holds them. The build is four kernels
// with a fixed order of every reduction, so the table is a pure function of
// the codebook.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "qamw_device.cuh"
#include "qamw_internal.h"

namespace qamw {

// The finest grid whose table fits the encode's shared memory with 16-bit
// offsets (lists + identity list < 65536 entries) for the shipped codebooks.
// G is odd, so that the encode finds a cell by rounding (search_cell); the
// records (8 G^2 bytes) and overflow lists fit the encode's shared memory
// beside its 16 warps' buffers and the codebook.
#ifndef QAMW_GRID_LARGE
#define QAMW_GRID_LARGE 137
#endif
#ifndef QAMW_GRID_MID
#define QAMW_GRID_MID 145
#endif
int search_grid(int N) { return N >= 2048 ? QAMW_GRID_LARGE : (N >= 64 ? QAMW_GRID_MID : 33); }

// Overflow entries (counts included) the table holds: 12288 for N >= 2048,
// 4096 for smaller codebooks (whose cells hold fewer centroids); sized so
// that records and overflow fit the encode's shared memory.
int64_t search_capacity(int N) { return N >= 2048 ? 12288 : 4096; }

static size_t image_bytes(int N) {
  const int G = search_grid(N);
  return ((size_t)G * G * 8 + (size_t)search_capacity(N) * 2 + 15) & ~size_t(15);
}

size_t search_table_bytes(int N) { return (size_t)kSearchImageOffset + image_bytes(N); }

namespace {

constexpr double kCellMargin = 1e-3;   // cell enlargement, in cells (covers fp32 rounding of the cell index)
constexpr double kTieSlack = 1e-5;     // relative slack on D(Q)^2
constexpr float kAxisA = 2.0f;         // T(x) = x / (a + |x|): cells about 1/4 as wide at 0 as near |x| = 2
constexpr int kListMax = 256;          // first-test members a warp prunes (shared-memory buffer per warp)
constexpr int kListThreads = 256;      // threads per CTA of the count and fill kernels (one warp per cell)

__global__ void table_header_kernel(const float *codebook, int N, int G, int64_t capacity, SearchHeader *h) {
  __shared__ float red[32];
  float m = 0.0f;
  for (int i = threadIdx.x; i < 2 * N; i += blockDim.x) m = fmaxf(m, fabsf(codebook[i]));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    const float L = r * 1.5f + 2.0f;
    const float UL = L / (kAxisA + L);
    h->magic = kSearchMagic;
    h->N = N;
    h->G = G;
    h->total = 0;
    h->a = kAxisA;
    h->UL = UL;
    h->inv_cw = (float)G / (2.0f * UL);
    h->L = L;
    h->image_bytes = 0;
    h->pad = 0;
    h->valid = 0;
    h->capacity = (int32_t)capacity;
  }
}

// Enlarged bounds of cell (ix, iy) in x, in fp64: the u-interval
// [k / inv_cw - UL, (k + 1) / inv_cw - UL] widened by the margin, mapped back
// through T^-1(u) = a u / (1 - |u|), and widened by a relative 1e-12 for the
// fp64 rounding of that map.
__device__ __forceinline__ double axis_inv(double a, double u) { return a * u / (1.0 - fabs(u)); }
__device__ __forceinline__ void cell_bounds(const SearchHeader &h, int cell, double &x0, double &x1, double &y0,
                                            double &y1) {
  const int ix = cell % h.G, iy = cell / h.G;
  const double a = (double)h.a, UL = (double)h.UL, cw = 1.0 / (double)h.inv_cw, m = kCellMargin * cw;
  const double lo_x = axis_inv(a, ix * cw - UL - m), hi_x = axis_inv(a, (ix + 1) * cw - UL + m);
  const double lo_y = axis_inv(a, iy * cw - UL - m), hi_y = axis_inv(a, (iy + 1) * cw - UL + m);
  x0 = lo_x - 1e-12 * fabs(lo_x);
  x1 = hi_x + 1e-12 * fabs(hi_x);
  y0 = lo_y - 1e-12 * fabs(lo_y);
  y1 = hi_y + 1e-12 * fabs(hi_y);
}

__device__ __forceinline__ double dmax2(double cx, double cy, double x0, double x1, double y0, double y1) {
  const double ax = fmax(fabs(cx - x0), fabs(cx - x1)), ay = fmax(fabs(cy - y0), fabs(cy - y1));
  return ax * ax + ay * ay;
}
__device__ __forceinline__ double dmin2(double cx, double cy, double x0, double x1, double y0, double y1) {
  const double ax = fmax(0.0, fmax(x0 - cx, cx - x1)), ay = fmax(0.0, fmax(y0 - cy, cy - y1));
  return ax * ax + ay * ay;
}

// D(Q)^2 * (1 + slack) for the warp's cell; every lane gets it.
__device__ double cell_bound(const float *codebook, int N, double x0, double x1, double y0, double y1, int lane) {
  double d = DBL_MAX;
  for (int i = lane; i < N; i += 32) d = fmin(d, dmax2(codebook[2 * i], codebook[2 * i + 1], x0, x1, y0, y1));
  for (int o = 16; o > 0; o >>= 1) d = fmin(d, __shfl_xor_sync(0xffffffffu, d, o));
  return d * (1.0 + kTieSlack);
}

// The members of the cell's first-test list, ascending, into the warp's buffer
// (when there are at most kListMax of them); returns their number.
__device__ int first_test(const float *codebook, int N, double x0, double x1, double y0, double y1, int lane,
                          uint16_t *buf) {
  const double bound = cell_bound(codebook, N, x0, x1, y0, y1, lane);
  int n = 0;
  for (int base = 0; base < N; base += 32) {
    const int i = base + lane;
    const bool in = i < N && dmin2(codebook[2 * i], codebook[2 * i + 1], x0, x1, y0, y1) <= bound;
    const uint32_t m = __ballot_sync(0xffffffffu, in);
    const int at = n + __popc(m & ((1u << lane) - 1u));
    if (in && at < kListMax) buf[at] = (uint16_t)i;
    n += __popc(m);
  }
  __syncwarp();
  return n;
}

// Whether member k of the buffer is beaten at all four corners of the cell by
// another member (the second test).
__device__ bool beaten(const float *codebook, const uint16_t *buf, int n, int k, double x0, double x1, double y0,
                       double y1) {
  const double px[4] = {x0, x0, x1, x1}, py[4] = {y0, y1, y0, y1};
  const int c = buf[k];
  const double cx = codebook[2 * c], cy = codebook[2 * c + 1];
  double dc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) dc[q] = (px[q] - cx) * (px[q] - cx) + (py[q] - cy) * (py[q] - cy);
  for (int j = 0; j < n; ++j) {
    if (j == k) continue;
    const int o = buf[j];
    const double ox = codebook[2 * o], oy = codebook[2 * o + 1];
    bool all = true;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double d = (px[q] - ox) * (px[q] - ox) + (py[q] - oy) * (py[q] - oy);
      all = all && (dc[q] > (1.0 + kTieSlack) * d);
    }
    if (all) return true;
  }
  return false;
}

// Per-cell list length (after pruning) into the record slot, as scratch.
__global__ void __launch_bounds__(kListThreads) table_count_kernel(const float *codebook, SearchHeader *h,
                                                                   uint64_t *rec) {
  __shared__ uint16_t bufs[kListThreads / 32][kListMax];
  const int lane = threadIdx.x & 31;
  uint16_t *buf = bufs[threadIdx.x >> 5];
  const int cell = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const SearchHeader hh = *h;
  if (cell >= hh.G * hh.G) return;
  double x0, x1, y0, y1;
  cell_bounds(hh, cell, x0, x1, y0, y1);
  const int n = first_test(codebook, hh.N, x0, x1, y0, y1, lane, buf);
  int cnt = n;
  if (n <= kListMax) {
    cnt = 0;
    for (int k = lane; k < n; k += 32) cnt += beaten(codebook, buf, n, k, x0, x1, y0, y1) ? 0 : 1;
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  }
  if (lane == 0) rec[cell] = (uint64_t)(uint32_t)cnt;
}

// Overflow offsets: a cell of count c > kSearchInline takes 1 + c - 3
// overflow entries (its extra count, then its entries beyond the third).
// Prefix sum in a fixed order (one CTA of 1024 threads); each thread owns up
// to kScanPer consecutive cells and writes rec[cell] = count | offset << 32.
constexpr int kScanPer = 32;   // up to 32768 cells (G <= kSearchMaxG) / 1024 threads
__device__ __forceinline__ uint32_t ovf_size(uint32_t c) { return c > (uint32_t)kSearchInline ? c - kSearchInline + 1 : 0u; }
__global__ void __launch_bounds__(1024) table_scan_kernel(SearchHeader *h, uint64_t *rec) {
  __shared__ uint32_t wsum[32];
  const int n = h->G * h->G;
  const int b = threadIdx.x * kScanPer;
  uint32_t cnt[kScanPer];
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    cnt[k] = (b + k < n) ? (uint32_t)rec[b + k] : 0u;
    s += ovf_size(cnt[k]);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = s;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0u;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  uint32_t run = inc - s + (warp > 0 ? wsum[warp - 1] : 0u);   // overflow entries before this thread's cells
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    if (b + k < n) {
      rec[b + k] = (uint64_t)cnt[k] | ((uint64_t)run << 32);
      run += ovf_size(cnt[k]);
    }
  }
  if (b < n && b + kScanPer >= n) {   // the thread that owns the last cell
    h->total = (int32_t)run;
    // offsets are 14-bit fields of the records
    h->valid = ((int64_t)run <= (int64_t)h->capacity && run < (1u << 14)) ? 1 : 0;
    h->image_bytes = (int32_t)(((size_t)n * 8 + (size_t)h->capacity * 2 + 15) & ~size_t(15));
  }
}

// The final records and overflow lists. The warp writes its list's entries by
// position: positions 0..2 into the record, later ones into the overflow.
__global__ void __launch_bounds__(kListThreads) table_fill_kernel(const float *codebook, const SearchHeader *h,
                                                                  uint64_t *rec, uint16_t *ovf) {
  __shared__ uint16_t bufs[kListThreads / 32][kListMax];
  __shared__ uint32_t heads[kListThreads / 32][kSearchInline];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint16_t *buf = bufs[wib];
  const int cell = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const SearchHeader hh = *h;
  if (!hh.valid || cell >= hh.G * hh.G) return;
  const uint64_t scratch = rec[cell];
  const uint32_t count = (uint32_t)scratch, off = (uint32_t)(scratch >> 32);
  double x0, x1, y0, y1;
  cell_bounds(hh, cell, x0, x1, y0, y1);
  const int n = first_test(codebook, hh.N, x0, x1, y0, y1, lane, buf);
  auto emit = [&](uint32_t pos, uint32_t idx) {
    if (pos < (uint32_t)kSearchInline) heads[wib][pos] = idx;
    else ovf[off + 1 + (pos - kSearchInline)] = (uint16_t)idx;
  };
  uint32_t pos = 0;
  if (n <= kListMax) {
    for (int base = 0; base < n; base += 32) {
      const int k = base + lane;
      const bool keep = k < n && !beaten(codebook, buf, n, k, x0, x1, y0, y1);
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) emit(pos + __popc(m & ((1u << lane) - 1u)), buf[k]);
      pos += __popc(m);
    }
  } else {   // too long to prune: the whole first-test list
    const double bound = cell_bound(codebook, hh.N, x0, x1, y0, y1, lane);
    for (int base = 0; base < hh.N; base += 32) {
      const int i = base + lane;
      const bool keep = i < hh.N && dmin2(codebook[2 * i], codebook[2 * i + 1], x0, x1, y0, y1) <= bound;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) emit(pos + __popc(m & ((1u << lane) - 1u)), (uint32_t)i);
      pos += __popc(m);
    }
  }
  __syncwarp();
  if (lane == 0) {
    // pos == count: both passes see the same lists
    const uint32_t e0 = heads[wib][0];
    const uint32_t e1 = count > 1 ? heads[wib][1] : e0, e2 = count > 2 ? heads[wib][2] : e0;
    uint32_t meta = count;
    if (count > (uint32_t)kSearchInline) {
      ovf[off] = (uint16_t)(count - kSearchInline);
      meta = off << 2;
    }
    rec[cell] = search_record(e0, e1, e2, meta);
  }
}

// Test hook: the encode's cell computation on given pairs.
__global__ void search_cells_kernel(const float *x, int64_t n, const SearchHeader *h, int32_t *cell_out) {
  const SearchHeader hh = *h;
  const bool ok = hh.magic == kSearchMagic && hh.valid == 1 && hh.G >= 1 && hh.G <= kSearchMaxG && (hh.G & 1) == 1;
  const float cbias = kCellMagic + (float)((hh.G - 1) / 2);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    cell_out[i] = ok ? search_cell(x[2 * i], x[2 * i + 1], hh.a, hh.inv_cw, cbias, hh.L, hh.G) : -1;
}

}  // namespace

cudaError_t launch_search_cells(const float *x, int64_t n, const void *table, int32_t *cell_out, cudaStream_t s) {
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4096);
  search_cells_kernel<<<(int)std::max<int64_t>(blocks, 1), 256, 0, s>>>(
      x, n, reinterpret_cast<const SearchHeader *>(table), cell_out);
  return cudaGetLastError();
}

cudaError_t launch_build_search_table(const float *codebook, int N, void *table, cudaStream_t s) {
  const int G = search_grid(N);
  SearchHeader *h = reinterpret_cast<SearchHeader *>(table);
  uint64_t *rec = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(table) + kSearchImageOffset);
  uint16_t *ovf = reinterpret_cast<uint16_t *>(rec + (size_t)G * G);
  table_header_kernel<<<1, 1024, 0, s>>>(codebook, N, G, search_capacity(N), h);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int cells = G * G;
  const int threads = kListThreads;
  const int blocks = (cells * 32 + threads - 1) / threads;
  table_count_kernel<<<blocks, threads, 0, s>>>(codebook, h, rec);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  table_scan_kernel<<<1, 1024, 0, s>>>(h, rec);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  table_fill_kernel<<<blocks, threads, 0, s>>>(codebook, h, rec, ovf);
  return cudaGetLastError();
}

}  // namespace qamw
