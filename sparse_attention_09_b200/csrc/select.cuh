// Streaming top-k candidate sets for the fused indexer (fine-grained token selection done on
// chip).  A "group" is 4 epilogue warps (128 threads) that share one named barrier; every
// function here is executed by all 128 threads of a group together.
//
// A token's candidate set is split into 4 regions of Q entries, one per warp of its group:
// a warp appends the candidates among its own 32 keys of a tile to its own region, with the
// fill count held in registers, so appending needs no atomics.  The regions are read
// together only at the (rare) cut points, where the survivors are spread round-robin over
// the regions again.
//
// Order: key (order-preserving uint32 of the fp32 score) descending, then index ascending.
// Candidates arrive in increasing index order from tile to tile.
#pragma once

#include "common.cuh"

namespace dsa {
namespace sel {

constexpr int kBuckets = 1024;

struct Group {
  int bar;  // named barrier id
  int tid;  // 0..127 inside the group
  __device__ __forceinline__ int warp() const { return tid >> 5; }
  __device__ __forceinline__ int lane() const { return tid & 31; }
};

__device__ __forceinline__ void gsync(const Group& G) {
  asm volatile("bar.sync %0, 128;" ::"r"(G.bar) : "memory");
}

// Barrier over the group that also ORs a predicate across it, so that a decision to leave a
// loop is the same in every thread (a named barrier cannot time out).
__device__ __forceinline__ bool gany(const Group& G, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %2, 0;\n\t"
      "bar.red.or.pred p, %1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(G.bar), "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Exclusive scan over the group; `scratch` holds 4 ints.
__device__ __forceinline__ int gscan(const Group& G, int v, int* scratch, int& total) {
  const int inc = warp_inclusive_scan(v);
  if (G.lane() == 31) scratch[G.warp()] = inc;
  gsync(G);
  const int w0 = scratch[0], w1 = scratch[1], w2 = scratch[2], w3 = scratch[3];
  total = w0 + w1 + w2 + w3;
  const int w = G.warp();
  const int wprefix = (w > 0 ? w0 : 0) + (w > 1 ? w1 : 0) + (w > 2 ? w2 : 0);
  gsync(G);
  return wprefix + inc - v;
}

struct Scratch {
  uint32_t hist[kBuckets];
  int scan[4];
  uint32_t bin, rem, eqcount, kmin, kmax, cursor, above;
  uint32_t tmp_key[128];
  int32_t tmp_idx[128];
};

struct Cands {
  uint32_t* key;  // [4 * Q]
  int32_t* idx;   // [4 * Q]
  int* cnt;       // [4] fill count of each region (valid at cut points)
  int Q;          // region capacity (<= 1152)
};

__device__ __forceinline__ int total_count(const Cands& C) { return C.cnt[0] + C.cnt[1] + C.cnt[2] + C.cnt[3]; }

// Histogram increment (a shared-memory reduction; lanes hitting one bin are combined by the
// memory unit).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
  if (valid) atomicAdd(&hist[bin], 1u);
}

// Calls f(key, idx, valid) for every entry of this warp's region, 32 at a time, with every
// lane of the warp taking part in each call.
template <class F>
__device__ __forceinline__ void for_region(const Group& G, const Cands& C, F f) {
  const int w = G.warp(), lane = G.lane();
  const int c = C.cnt[w];
  const uint32_t* kp = C.key + w * C.Q;
  const int32_t* ip = C.idx + w * C.Q;
  int i0 = 0;
  for (; i0 + 32 < c; i0 += 64) {  // two entries per lane in flight
    const int i = i0 + lane, j = i0 + 32 + lane;
    const bool vj = j < c;
    const uint32_t ka = kp[i], kb = vj ? kp[j] : 0u;
    const int32_t ia = ip[i], ib = vj ? ip[j] : 0;
    f(ka, ia, true);
    f(kb, ib, vj);
  }
  for (; i0 < c; i0 += 32) {
    const int i = i0 + lane;
    const bool v = i < c;
    f(v ? kp[i] : 0u, v ? ip[i] : 0, v);
  }
}

// Group-wide minimum and maximum of per-thread values.
__device__ __forceinline__ void group_minmax(const Group& G, Scratch& S, uint32_t mn, uint32_t mx, uint32_t& omn,
                                             uint32_t& omx) {
  if (G.tid == 0) {
    S.kmin = 0xFFFFFFFFu;
    S.kmax = 0u;
  }
  gsync(G);
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (G.lane() == 0) {
    atomicMin(&S.kmin, mn);
    atomicMax(&S.kmax, mx);
  }
  gsync(G);
  omn = S.kmin;
  omx = S.kmax;
  gsync(G);
}

// Keeps the entries with keep(key, idx), spreads them round-robin over the 4 regions and
// returns the smallest kept key.  Every entry of the warp's region is read into registers
// before the barrier that precedes the first write, so no entry is overwritten unread.  The
// order of entries inside a set carries no meaning (emission goes through a bitmap, cuts rank
// by key and index), so each lane's kept entries take consecutive output positions: one warp
// scan and one group scan place them (no shared-memory atomics, no per-round ballots).
template <class Keep>
__device__ __forceinline__ uint32_t compact(const Group& G, const Cands& C, Scratch& S, Keep keep) {
  constexpr int kMaxRounds = 36;  // Q <= 1152 = 32 lanes x 36 rounds
  const int w = G.warp(), lane = G.lane();
  // the set's fields in registers: stores through its pointers cannot then force reloads of
  // the descriptor (which the compiler must otherwise assume they may overwrite)
  uint32_t* const ckey = C.key;
  int32_t* const cidx = C.idx;
  int* const ccnt = C.cnt;
  const int Q = C.Q;
  const int c = ccnt[w];
  uint32_t key[kMaxRounds];
  int32_t id[kMaxRounds];
  uint64_t keepbits = 0u;  // bit r: this lane keeps its entry of round r
#pragma unroll
  for (int r = 0; r < kMaxRounds; ++r) {
    const int i = r * 32 + lane;
    key[r] = 0u;
    id[r] = 0;
    if (i < c) {
      key[r] = ckey[w * Q + i];
      id[r] = cidx[w * Q + i];
      if (keep(key[r], id[r])) keepbits |= 1ull << r;
    }
  }
  const int mine = __popcll(keepbits);
  const int incl = warp_inclusive_scan(mine);
  const int wcount = __shfl_sync(0xffffffffu, incl, 31);
  int total;
  int base = gscan(G, lane == 0 ? wcount : 0, S.scan, total);  // its barriers order reads before writes
  base = __shfl_sync(0xffffffffu, base, 0);
  uint32_t p = static_cast<uint32_t>(base + incl - mine);
  uint32_t mn = 0xFFFFFFFFu;
#pragma unroll
  for (int r = 0; r < kMaxRounds; ++r) {
    if ((keepbits >> r) == 0ull) break;
    if ((keepbits >> r) & 1ull) {
      const int slot = static_cast<int>(p & 3u) * Q + static_cast<int>(p >> 2);
      ckey[slot] = key[r];
      cidx[slot] = id[r];
      mn = min(mn, key[r]);
      ++p;
    }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  if (lane == 0) S.tmp_key[w] = mn;  // tmp_key is free here (cut_final is done with it)
  gsync(G);
  const uint32_t kmin = min(min(S.tmp_key[0], S.tmp_key[1]), min(S.tmp_key[2], S.tmp_key[3]));
  if (G.tid < 4) ccnt[G.tid] = total / 4 + (G.tid < total % 4 ? 1 : 0);
  gsync(G);  // every thread has read tmp_key and C.cnt is published before anyone moves on
  return kmin;
}

// Warp 0 of the group: walk 256 bins from the top (descending) or the bottom and find where
// the running count reaches `want`; writes S.bin, S.rem (still needed inside the bin) and
// S.eqcount.
__device__ __forceinline__ void find_bin256(const Group& G, Scratch& S, uint32_t want, bool descending) {
  const int lane = G.lane();
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int bin = descending ? 255 - (8 * lane + j) : 8 * lane + j;
    c[j] = S.hist[bin];
    sum += c[j];
  }
  const uint32_t inc = static_cast<uint32_t>(warp_inclusive_scan(static_cast<int>(sum)));
  const uint32_t before = inc - sum;
  if (before < want && want <= inc) {
    uint32_t acc = before;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (acc + c[j] >= want) {
        S.bin = descending ? 255u - static_cast<uint32_t>(8 * lane + j) : static_cast<uint32_t>(8 * lane + j);
        S.rem = want - acc;
        S.eqcount = c[j];
        break;
      }
      acc += c[j];
    }
  }
}

// Exact cut to the m best by radix select (key, then index among equal keys).  Used when
// many candidates share one key.  Requires 1 <= m < total_count.  Returns the smallest kept key.
__device__ __noinline__ uint32_t cut_exact(const Group G, const Cands C, Scratch& S, int m) {
  const int tid = G.tid;
  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(m);
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    S.hist[tid] = 0u;
    S.hist[tid + 128] = 0u;
    gsync(G);
    for_region(G, C, [&](uint32_t key, int32_t, bool v) {
      hist_add(S.hist, (key >> shift) & 255u, v && (key & mask) == prefix);
    });
    gsync(G);
    if (G.warp() == 0) find_bin256(G, S, remaining, true);
    gsync(G);
    prefix |= S.bin << shift;
    mask |= 255u << shift;
    remaining = S.rem;
    gsync(G);
  }
  const uint32_t kth = prefix, need_eq = remaining;
  uint32_t idx_thr = 0xFFFFFFFFu;  // keep every equal key unless there are more than needed
  if (S.eqcount != need_eq) {
    uint32_t iprefix = 0, imask = 0, irem = need_eq;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {  // indices < 2^24
      const int shift = 16 - 8 * pass;
      S.hist[tid] = 0u;
      S.hist[tid + 128] = 0u;
      gsync(G);
      for_region(G, C, [&](uint32_t key, int32_t id, bool v) {
        const uint32_t u = static_cast<uint32_t>(id);
        hist_add(S.hist, (u >> shift) & 255u, v && key == kth && (u & imask) == iprefix);
      });
      gsync(G);
      if (G.warp() == 0) find_bin256(G, S, irem, false);
      gsync(G);
      iprefix |= S.bin << shift;
      imask |= 255u << shift;
      irem = S.rem;
      gsync(G);
    }
    idx_thr = iprefix;
  }
  return compact(G, C, S, [=](uint32_t key, int32_t id) {
    return key > kth || (key == kth && static_cast<uint32_t>(id) <= idx_thr);
  });
}

// Buckets of a key range [lo, hi]: key -> (key - lo) >> shift, with the smallest shift that
// leaves at most kBuckets buckets (kBuckets is a power of two).  Bucket b holds exactly the keys
// [lo + (b << shift), lo + ((b + 1) << shift) - 1], so a bucket's bounds are exact and the keys
// of a bucket and everything above it are those >= its smallest key.
__device__ __forceinline__ int bucket_shift(uint32_t lo, uint32_t hi) {
  const uint32_t span = hi - lo;
  const int bits = 32 - __clz(span);  // bits of the largest offset
  constexpr int kBucketBits = 10;
  static_assert((1 << kBucketBits) == kBuckets, "kBuckets is 2^kBucketBits");
  return bits > kBucketBits ? bits - kBucketBits : 0;
}

struct Boundary {
  uint32_t lo, hi;  // the boundary bucket's keys: exactly [lo, hi]
  int above;        // candidates ranked above the boundary bucket
  int inb;          // candidates in the boundary bucket
};

// One histogram round over the candidates with keys in [lo, hi]: finds the bucket where the
// count from the top reaches `want` (counting `above_in` candidates already known to be
// larger than hi, plus those found above hi in this pass).
__device__ __forceinline__ Boundary boundary_round(const Group& G, const Cands& C, Scratch& S, uint32_t lo,
                                                   uint32_t hi, int want) {
  const int tid = G.tid;
  const int shift = bucket_shift(lo, hi);
#pragma unroll
  for (int i = 0; i < kBuckets / 128; ++i) S.hist[tid * (kBuckets / 128) + i] = 0u;
  if (tid == 0) S.above = 0u;
  gsync(G);
  uint32_t above = 0;
  for_region(G, C, [&](uint32_t key, int32_t, bool v) {
    const bool in = v && key >= lo && key <= hi;
    above += (v && key > hi) ? 1u : 0u;
    hist_add(S.hist, in ? (key - lo) >> shift : 0u, in);
  });
  above = __reduce_add_sync(0xffffffffu, above);
  if (G.lane() == 0) atomicAdd(&S.above, above);
  gsync(G);
  constexpr int PER = kBuckets / 128;  // thread i owns buckets kBuckets-1-PER*i-(PER-1) .. kBuckets-1-PER*i
  uint32_t c[PER], sum = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = S.hist[kBuckets - 1 - (PER * tid + j)];
    sum += c[j];
  }
  int total;
  const uint32_t above_hi = S.above;
  const uint32_t before = above_hi + static_cast<uint32_t>(gscan(G, static_cast<int>(sum), S.scan, total));
  const uint32_t wnt = static_cast<uint32_t>(want);
  if (before < wnt && wnt <= before + sum) {
    uint32_t acc = before;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (acc + c[j] >= wnt) {
        S.bin = static_cast<uint32_t>(kBuckets - 1 - (PER * tid + j));
        S.rem = acc;
        S.eqcount = c[j];
        break;
      }
      acc += c[j];
    }
  }
  gsync(G);
  Boundary b;
  b.above = static_cast<int>(S.rem);
  b.inb = static_cast<int>(S.eqcount);
  b.lo = lo + (S.bin << shift);
  const uint64_t top = static_cast<uint64_t>(b.lo) + ((1ull << shift) - 1u);
  b.hi = top < hi ? static_cast<uint32_t>(top) : hi;
  gsync(G);
  return b;
}

// Streaming cut, run when a region is about to overflow.  Keeps a superset of the current
// top k (the boundary bucket and everything above it) when that leaves at most `limit`
// entries; otherwise narrows the interval and retries, and at last cuts exactly.  [lo, hi]
// bounds the keys of the set.  Returns the new acceptance threshold (the smallest kept key):
// later keys enter only if key > thr, which is exact because later candidates have larger
// indices than every kept one and at least k kept candidates are >= the smallest kept key.
__device__ __noinline__ uint32_t cut_stream(const Group G, const Cands C, Scratch& S, int k, int limit, uint32_t lo,
                                            uint32_t hi) {
  const int n = total_count(C);
  uint32_t rlo = lo, rhi = hi;
#pragma unroll 1
  for (int round = 0; round < 3; ++round) {
    const Boundary bd = boundary_round(G, C, S, rlo, rhi, k);
    const int kept = bd.above + bd.inb;
    if (kept <= limit && kept < n) {  // keep the boundary bucket and everything above it
      const uint32_t kf = bd.lo;
      return compact(G, C, S, [=](uint32_t key, int32_t) { return key >= kf; });
    }
    if (bd.lo >= bd.hi || (bd.lo == rlo && bd.hi == rhi)) break;
    rlo = bd.lo;
    rhi = bd.hi;
  }
  return cut_exact(G, C, S, k);
}

// Final exact cut to the m best (key descending, index ascending).
__device__ __noinline__ void cut_final(const Group G, const Cands C, Scratch& S, int m, uint32_t lo, uint32_t hi) {
  const int n = total_count(C);
  if (n <= m) return;
  uint32_t rlo = lo, rhi = hi;
  Boundary bd;
  bool found = false;
#pragma unroll 1
  for (int round = 0; round < 3; ++round) {
    bd = boundary_round(G, C, S, rlo, rhi, m);
    if (bd.inb <= 128) {
      found = true;
      break;
    }
    if (bd.lo >= bd.hi || (bd.lo == rlo && bd.hi == rhi)) break;
    rlo = bd.lo;
    rhi = bd.hi;
  }
  if (!found) {  // many equal keys: resolve by index with the radix path
    cut_exact(G, C, S, m);
    return;
  }
  const int need = m - bd.above;  // 1 <= need <= inb
  const uint32_t blo = bd.lo, bhi = bd.hi;
  auto in_bucket = [=](uint32_t key) { return key >= blo && key <= bhi; };
  if (need == bd.inb) {  // the whole boundary bucket and everything above it
    compact(G, C, S, [=](uint32_t key, int32_t) { return key >= blo; });
    return;
  }
  // gather the boundary bucket and find its need-th best by ranking
  const int tid = G.tid;
  if (tid == 0) S.rem = 0u;
  gsync(G);
  for_region(G, C, [&](uint32_t key, int32_t id, bool v) {
    if (v && in_bucket(key)) {
      const int pos = static_cast<int>(atomicAdd(&S.rem, 1u));
      S.tmp_key[pos] = key;
      S.tmp_idx[pos] = id;
    }
  });
  gsync(G);
  if (tid < bd.inb) {
    const uint32_t kj = S.tmp_key[tid];
    const int32_t ij = S.tmp_idx[tid];
    int rank = 0;
    for (int i = 0; i < bd.inb; ++i) rank += (S.tmp_key[i] > kj || (S.tmp_key[i] == kj && S.tmp_idx[i] < ij)) ? 1 : 0;
    if (rank == need - 1) {
      S.bin = kj;
      S.eqcount = static_cast<uint32_t>(ij);
    }
  }
  gsync(G);
  // the m-th best is (kstar, istar): every key above the boundary bucket is > kstar (buckets are
  // monotone) and every key below it < kstar, so the m best are those ranked at or before it
  const uint32_t kstar = S.bin, istar = S.eqcount;
  compact(G, C, S, [=](uint32_t key, int32_t id) {
    return key > kstar || (key == kstar && static_cast<uint32_t>(id) <= istar);
  });
}

// Writes the (already cut) set to out[0..k) in ascending index order, -1 padded.  `bitmap`
// has room for `positions` bits.
__device__ __noinline__ void emit_sorted(const Group G, const Cands C, Scratch& S, uint32_t* bitmap, int positions,
                                         int32_t* out, int k) {
  const int tid = G.tid, warp = G.warp(), lane = G.lane();
  const int nwords = (positions + 31) / 32;
  for (int wd = tid; wd < nwords; wd += 128) bitmap[wd] = 0u;
  gsync(G);
  for_region(G, C, [&](uint32_t, int32_t id, bool v) {
    if (v) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
  });
  gsync(G);
  // warp w owns 32-word chunks [w*per, (w+1)*per); lane l reads word chunk*32 + l
  const int nchunks = (nwords + 31) / 32;
  const int per = (nchunks + 3) / 4;
  const int c0 = min(nchunks, warp * per), c1 = min(nchunks, c0 + per);
  int bits = 0;
  for (int c = c0; c < c1; ++c) {
    const int wd = c * 32 + lane;
    bits += wd < nwords ? __popc(bitmap[wd]) : 0;
  }
  bits = __reduce_add_sync(0xffffffffu, bits);
  int total;
  int pos = gscan(G, lane == 0 ? bits : 0, S.scan, total);
  pos = __shfl_sync(0xffffffffu, pos, 0);
  for (int c = c0; c < c1; ++c) {
    const int wd = c * 32 + lane;
    uint32_t word = wd < nwords ? bitmap[wd] : 0u;
    const int cnt = __popc(word);
    const int inc = warp_inclusive_scan(cnt);
    int o = pos + inc - cnt;
    while (word) {
      const int bit = __ffs(word) - 1;
      out[o++] = wd * 32 + bit;
      word &= word - 1;
    }
    pos += __shfl_sync(0xffffffffu, inc, 31);
  }
  for (int i = total + tid; i < k; i += 128) out[i] = -1;
  gsync(G);
}

}  // namespace sel
}  // namespace dsa
