// ivf.cuh -- inverted lists of an IVF coarse quantizer from a top-m assignment.
//
// "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering",
// abstract: the mixture is the coarse quantizer of an IVF index, and its
// responsibilities file a vector that lies near a cluster border under more
// than one cluster.  The pages give no rule; the one built here: point n joins
// the list of its most responsible component always, and the list of its
// rank-j component (j >= 2) when that responsibility is >= tau (compared in
// float32).  The lists are compressed rows -- list k is
// ids[offsets[k] .. offsets[k+1]) -- with point indices ascending inside each
// list, so the result is deterministic.
//
// A stable counting sort in three steps, all plain loads and stores (the work
// is a few bytes per point; HBM-bound, nothing for the tensor cores):
//   1. count: the points are cut into B contiguous chunks, one warp per chunk.
//      The warp walks its chunk 32 points at a time, in order, and adds each
//      list's entries to cnt[k * B + c] (list-major, so step 2 reads each list's
//      counts contiguously).
//   2. scan:  per list, the exclusive prefix of its counts over the chunks (in
//      place) and the list's total; then one block turns the totals into
//      offsets.
//   3. fill:  each warp walks its chunk again with the same code, now writing
//      every kept point to offsets[k] + cnt[k * B + c] + (entries of list k
//      from lower lanes of the same 32-point group).
// Inside a 32-point group the rank of an entry among the group's entries of
// the same list comes from a small per-warp hash table in shared memory (a
// point's m components are distinct, so each list takes at most one entry per
// point); the lane holding a list's last entry in the group advances that
// list's counter.  One warp owns each counter column, so the counters need no
// global atomics and the order is fixed.  Where K is small the running counts
// live in the warp's shared memory and reach cnt once per chunk.
#pragma once
#include <algorithm>

#include "common.cuh"

namespace scem {

constexpr int kIvfWarps = 8;                          // warps (chunks) per CTA
constexpr int64_t kIvfMinPoints = 256;                // points per chunk, at least
constexpr int64_t kIvfMaxChunks = 148 * 8;            // one CTA of 8 warps per SM (measured)
constexpr size_t kIvfCountBytes = (size_t)64 << 20;   // bound on the count matrix

// Workspace of gmm_ivf_build:
//   status : uint32 device status word (GMM_DEVFLAG_BAD_INDEX), 256 bytes
//   tot    : K int64, list sizes
//   cnt    : K x B int64, per-chunk counts of each list, then their prefixes
struct IvfLayout {
  size_t status, tot, cnt, total;
  int B;       // chunks
  int64_t R;   // points per chunk (the last ones may hold fewer, or none)
};

inline IvfLayout ivf_layout(int64_t N, int K) {
  IvfLayout L;
  int64_t b = (N + kIvfMinPoints - 1) / kIvfMinPoints;
  b = std::min(b, kIvfMaxChunks);
  b = std::min(b, std::max<int64_t>(1, (int64_t)(kIvfCountBytes / ((size_t)K * 8))));
  L.B = (int)std::max<int64_t>(b, 1);
  L.R = (N + L.B - 1) / L.B;
  size_t off = 0;
  L.status = off;
  off = 256;
  L.tot = off;
  off = align_up(off + (size_t)K * 8, 256);
  L.cnt = off;
  off = align_up(off + (size_t)L.B * K * 8, 256);
  L.total = off;
  return L;
}

// Slots of a warp's hash table: a power of two at least twice the 32 * m
// entries of a group, so an insertion always finds its key or an empty slot.
constexpr int ivf_table_log2(int m) { return m <= 1 ? 6 : m <= 2 ? 7 : m <= 4 ? 8 : 9; }

// Steps 1 (kFill = false) and 3 (kFill = true), for m = kM candidates per point.
// An index outside [0, K), or one that repeats an earlier index of the same
// point, is skipped and raises GMM_DEVFLAG_BAD_INDEX; both passes skip the
// same entries.
//
// Ranks inside a group: every kept entry inserts its list into the warp's
// shared-memory hash table (open addressing, atomicCAS) and ORs its lane bit
// into that slot's mask, so after one __syncwarp a slot's mask is the set of
// lanes holding that list; the entry's rank is the count of mask bits below
// its lane.  The masks do not depend on the order of the atomics, so neither
// does the result.
//
// kShared (K small enough, see ivf_shared_counters): each warp keeps its
// chunk's running count of every list in shared memory (int32, from 0) instead
// of in cnt, so no global load and store sits on the per-group chain.  The
// count pass writes the final counts to cnt once at the end; the fill pass
// reads each entry's chunk prefix from cnt (read-only there) and adds the
// shared count.
template <int kM, bool kFill, bool kShared>
__global__ void __launch_bounds__(kIvfWarps * 32, kM <= 4 ? 4 : 2)
    ivf_walk_kernel(int64_t N, int K, const int32_t* __restrict__ idx,
                    const float* __restrict__ resp, float tau, int B, int64_t R, int64_t* cnt,
                    const int64_t* __restrict__ offsets, int64_t* __restrict__ ids,
                    unsigned int* status) {
  constexpr int kLog = ivf_table_log2(kM);
  constexpr int kT = 1 << kLog;
  __shared__ int s_key[kIvfWarps][kT];
  __shared__ unsigned int s_lanes[kIvfWarps][kT];
  extern __shared__ int ivf_counts[];  // kShared: [kIvfWarps][K]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * kIvfWarps + w;
  if (c >= B) return;  // c is the same for the whole warp; the tables are per warp
  int* key = s_key[w];
  unsigned int* lanes = s_lanes[w];
  for (int i = lane; i < kT; i += 32) {
    key[i] = -1;
    lanes[i] = 0u;
  }
  int* scnt = ivf_counts + (size_t)w * K;
  if (kShared)
    for (int k = lane; k < K; k += 32) scnt[k] = 0;
  __syncwarp();
  const unsigned int below = (1u << lane) - 1u;
  const unsigned int above = ~below & ~(1u << lane);
  const int64_t lo = min(N, (int64_t)c * R);
  const int64_t hi = min(N, lo + R);
  bool bad = false;
  // the group's indices and responsibilities, loaded one group ahead
  int nv[kM];
  float nr[kM];
  auto load = [&](int64_t n) {
#pragma unroll
    for (int j = 0; j < kM; ++j) {
      nv[j] = n < hi ? idx[n * kM + j] : -1;
      nr[j] = (j > 0 && n < hi) ? resp[n * kM + j] : 0.f;
    }
  };
  load(lo + lane);
  for (int64_t g = lo; g < hi; g += 32) {  // the same trip count for every lane
    const int64_t n = g + lane;
    int v[kM];
    float r[kM];
#pragma unroll
    for (int j = 0; j < kM; ++j) {
      v[j] = nv[j];
      r[j] = nr[j];
    }
    load(n + 32);
    int e[kM];     // kept list of each rank, -1 if none
    int slot[kM];  // its slot in the table
#pragma unroll
    for (int j = 0; j < kM; ++j) {
      e[j] = -1;
      slot[j] = 0;
      if (n < hi) {
        bool ok = v[j] >= 0 && v[j] < K;
#pragma unroll
        for (int i = 0; i < j; ++i) ok = ok && v[i] != v[j];
        bad |= !ok;
        if (ok && (j == 0 || r[j] >= tau)) e[j] = v[j];
      }
      if (e[j] >= 0) {
        unsigned int h = ((unsigned int)e[j] * 2654435761u) >> (32 - kLog);
        for (int probe = 0; probe < kT; ++probe) {  // ends at the first probe that fits
          const int old = atomicCAS(&key[h], -1, e[j]);
          if (old == -1 || old == e[j]) break;
          h = (h + 1) & (kT - 1);
        }
        slot[j] = (int)h;
        atomicOr(&lanes[h], 1u << lane);
      }
    }
    __syncwarp();  // every entry of the group is in the table
    int64_t base[kM];
    int before[kM];
    bool last[kM];
#pragma unroll
    for (int j = 0; j < kM; ++j) {
      const unsigned int mask = e[j] >= 0 ? lanes[slot[j]] : 0u;
      before[j] = __popc(mask & below);
      last[j] = (mask & above) == 0u;
      base[j] = e[j] < 0 ? 0 : kShared ? (int64_t)scnt[e[j]] : cnt[(int64_t)e[j] * B + c];
    }
    __syncwarp();  // every lane has read its mask and counter
#pragma unroll
    for (int j = 0; j < kM; ++j) {
      if (e[j] >= 0) {
        const int64_t rel = base[j] + before[j];
        if (kFill) {
          const int64_t pre = kShared ? cnt[(int64_t)e[j] * B + c] : 0;  // the chunk's prefix
          ids[offsets[e[j]] + pre + rel] = n;
        }
        if (last[j]) {
          if (kShared)
            scnt[e[j]] = (int)(rel + 1);
          else
            cnt[(int64_t)e[j] * B + c] = rel + 1;
        }
        key[slot[j]] = -1;
        lanes[slot[j]] = 0u;
      }
    }
    __syncwarp();  // counters advanced and the table empty for the next group
  }
  if (kShared && !kFill)
    for (int k = lane; k < K; k += 32) cnt[(int64_t)k * B + c] = scnt[k];
  if (bad) atomicOr(status, GMM_DEVFLAG_BAD_INDEX);
}

// Shared-memory counters: one int32 per list per warp, at most 64 KB per CTA,
// and a chunk's entries (R points times m) within int32.
inline bool ivf_shared_counters(int K, int64_t R, int m) {
  return (size_t)K * kIvfWarps * 4 <= (64u << 10) && R * m < ((int64_t)1 << 31);
}

// Step 2a: one warp per list; exclusive prefix of cnt[k * B + 0 .. B) in place,
// the list's size into tot[k].
__global__ void __launch_bounds__(kIvfWarps * 32)
    ivf_scan_chunks_kernel(int K, int B, int64_t* __restrict__ cnt, int64_t* __restrict__ tot) {
  const int lane = threadIdx.x & 31;
  const int k = blockIdx.x * kIvfWarps + (threadIdx.x >> 5);
  if (k >= K) return;  // k is the same for the whole warp
  int64_t* col = cnt + (int64_t)k * B;
  int64_t run = 0;
  for (int c0 = 0; c0 < B; c0 += 32) {
    const int c = c0 + lane;
    const int64_t v = c < B ? col[c] : 0;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (c < B) col[c] = run + x - v;
    run += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) tot[k] = run;
}

// Step 2b: one block of kIvfScanThreads; offsets[0..K] = exclusive prefix of
// tot, offsets[K] = the number of entries.
constexpr int kIvfScanThreads = 1024;

__global__ void __launch_bounds__(kIvfScanThreads)
    ivf_offsets_kernel(int K, const int64_t* __restrict__ tot, int64_t* __restrict__ offsets) {
  __shared__ int64_t wsum[kIvfScanThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (K + kIvfScanThreads - 1) / kIvfScanThreads;
  const int b = min(K, t * per), e = min(K, b + per);
  int64_t s = 0;
  for (int i = b; i < e; ++i) s += tot[i];
  int64_t x = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int64_t w = wsum[lane];
    int64_t y = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    wsum[lane] = y - w;  // warps before this one
  }
  __syncthreads();
  int64_t run = wsum[warp] + x - s;
  for (int i = b; i < e; ++i) {
    offsets[i] = run;
    run += tot[i];
  }
  if (t == kIvfScanThreads - 1) offsets[K] = run;
}

}  // namespace scem
