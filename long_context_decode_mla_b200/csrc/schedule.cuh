// Work schedule shared by the tensor-core decode kernels: which 64-row tiles
// a CTA processes, in which order, and where each request's piece of the
// result goes.  Integer bookkeeping only.
//
// Dense mode: the local tokens of all requests are cut into 64-row tiles (one
// cache block each) and laid end to end; CTA c owns tiles
// [c * tpc, (c + 1) * tpc) (common.cuh).  The tiles of one request inside
// that range form a segment.  Sparse mode: one CTA per (request, index-list
// chunk); the chunk is compacted to the local rows this shard owns and forms
// the CTA's single segment.
//
// The control structure passed as `Ctl` provides `int sel_count`,
// `int warp_sums[16]` and `Segment seg[kSchedMaxSeg]` in shared memory.
#pragma once

#include "common.cuh"

namespace dcpmla {

constexpr int kSchedMaxSeg = 128;   // segments collected per batch
constexpr int kTileRows = 64;       // rows per tile: one cache block

struct SegView {
  int b;
  int row_begin;   // first local row (dense); 0 (sparse, rows come from the list)
  int nrows;
  int ntiles;
  bool whole;      // the segment is the whole request: write the final result
};

template <class Ctl>
__device__ __forceinline__ SegView seg_view(const PartialParams& p, const Ctl& c, int k) {
  SegView v;
  if (p.sparse_idx) {
    v.b = blockIdx.x / p.sparse_parts;
    v.row_begin = 0;
    v.nrows = c.sel_count;
    v.whole = p.sparse_parts == 1;
  } else {
    const Segment s = c.seg[k];
    v.b = s.b;
    v.row_begin = s.t0 * kBlock;
    v.nrows = min(s.n_rows, s.t1 * kBlock) - v.row_begin;
    v.whole = s.t0 == 0 && s.t1 == s.nt;
  }
  v.ntiles = (v.nrows + kTileRows - 1) / kTileRows;
  return v;
}

// Workspace (or output) slot of a segment's result: the request itself when
// the segment is the whole request, else a split slot (dense: CTA + request,
// which is unique along the tile order; sparse: the CTA).
__device__ __forceinline__ size_t seg_slot(const PartialParams& p, const SegView& v) {
  if (v.whole) return (size_t)v.b;
  return p.sparse_idx ? (size_t)blockIdx.x : (size_t)blockIdx.x + v.b;
}

// Walks the CTA's tiles in order: segment k, tile t (segments without tiles
// are skipped).  Returns false past the last tile.
struct TileCursor {
  int k, t, nseg;
  SegView v;
  template <class Ctl>
  __device__ __forceinline__ bool start(const PartialParams& p, const Ctl& c, int n) {
    nseg = n;
    k = 0;
    t = 0;
    while (k < nseg) {
      v = seg_view(p, c, k);
      if (v.ntiles > 0) return true;
      ++k;
    }
    return false;
  }
  template <class Ctl>
  __device__ __forceinline__ bool next(const PartialParams& p, const Ctl& c) {
    if (++t < v.ntiles) return true;
    t = 0;
    while (++k < nseg) {
      v = seg_view(p, c, k);
      if (v.ntiles > 0) return true;
    }
    return false;
  }
  __device__ __forceinline__ bool last_of_segment() const { return t == v.ntiles - 1; }
  // valid rows of the current tile (64 except in a segment's last tile)
  __device__ __forceinline__ int tile_valid_rows() const {
    return min(kTileRows, v.nrows - t * kTileRows);
  }
};

// Collect this CTA's dense segments number [first, first + maxseg) in
// request order into c.seg (which holds maxseg entries).  Returns the total
// number of segments of the CTA.  All threads of the block call it.
template <class Ctl>
__device__ int collect_segments_n(const PartialParams& p, int lo, int hi, int first, int maxseg,
                                  Ctl& c) {
  int off = 0, seen = 0;
  for (int base = 0; base < p.batch && off < hi; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int n = 0, nt = 0;
    if (b < p.batch) nt = request_tiles(p, b, &n);
    int tot;
    const int start = off + block_exclusive_scan(nt, c.warp_sums, &tot);
    const int inter = (nt > 0 && start < hi && start + nt > lo) ? 1 : 0;
    int tot_inter;
    const int idx = seen + block_exclusive_scan(inter, c.warp_sums, &tot_inter);
    if (inter && idx >= first && idx < first + maxseg) {
      Segment s;
      s.b = b;
      s.t0 = max(lo, start) - start;
      s.t1 = min(hi, start + nt) - start;
      s.n_rows = n;
      s.nt = nt;
      c.seg[idx - first] = s;
    }
    seen += tot_inter;
    off += tot;
  }
  __syncthreads();
  return seen;
}

template <class Ctl>
__device__ int collect_segments(const PartialParams& p, int lo, int hi, int first, Ctl& c) {
  return collect_segments_n(p, lo, hi, first, kSchedMaxSeg, c);
}

// Sparse mode: this CTA's chunk of the index list, filtered to the positions
// this shard owns, as local indices (in list order) into `list`.  All threads
// of the block call it.
template <class Ctl>
__device__ int compact_sparse(const PartialParams& p, int* list, Ctl& c) {
  const int b = blockIdx.x / p.sparse_parts, part = blockIdx.x % p.sparse_parts;
  const int chunk = (p.topk + p.sparse_parts - 1) / p.sparse_parts;
  const int i0 = part * chunk, i1 = min(p.topk, i0 + chunk);
  int L = seq_len_of(p, b);
  if (L < 0) {
    if (threadIdx.x == 0 && p.flags) atomicOr(p.flags, kFlagBadLength);
    L = 0;
  }
  int count = 0;
  for (int base = i0; base < i1; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int sel = 0, j = 0;
    if (i < i1) {
      const int t = __ldg(p.sparse_idx + (size_t)b * p.topk + i);
      if (t >= 0 && t < L && t % p.nshards == p.shard) {
        j = t / p.nshards;
        if ((j >> 6) < p.bt_stride) {
          sel = 1;
        } else if (p.flags) {
          atomicOr(p.flags, kFlagBadLength);
        }
      }
    }
    int tot;
    const int pos = count + block_exclusive_scan(sel, c.warp_sums, &tot);
    if (sel) list[pos] = j;
    count += tot;
  }
  __syncthreads();
  return count;
}

}  // namespace dcpmla
