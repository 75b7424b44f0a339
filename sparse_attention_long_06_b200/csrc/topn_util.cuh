// Warp-level top-n block selection (step 4), shared by the prefill and
// decode kernels.
//
// Candidates are blocks j < ncand; the complete ones (j < ncmp) carry their
// score, the incomplete block holding the query competes with score 0.  The
// n largest under (score descending, index ascending) are found by an 8-bit
// radix select on an order-preserving 32-bit key of each score, followed by
// taking the lowest-index ties at the threshold.  The result is written in
// ascending block order, padded with -1.
#pragma once
#include <cstdint>

namespace nsa {

// Order-preserving key of an fp32 score: larger score, larger key; -0 and +0
// share a key (they compare equal); non-negative scores keep their bit
// pattern with the top bit set, negative ones are bit-inverted.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  b = (b == 0x80000000u) ? 0u : b;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
constexpr uint32_t kZeroScoreKey = 0x80000000u;  // score_key(0.f)

// `score(j)` returns the fp32 score of complete block j; `hist` is 256
// words of warp-private shared memory; `out(i, j)` stores result i.
template <typename ScoreFn, typename OutFn>
__device__ __forceinline__ void warp_topn(ScoreFn score, int ncmp, int ncand, int n,
                                          unsigned* hist, OutFn out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  auto bits = [&](int j) -> uint32_t { return j < ncmp ? score_key(score(j)) : kZeroScoreKey; };
  if (ncand <= n) {
    for (int j = lane; j < n; j += 32) out(j, j < ncand ? j : -1);
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  int k = n;  // rank still to be found inside the current prefix class
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hist[i] = 0;
    __syncwarp();
    // warp-aggregated counting: the lanes holding the same digit add their
    // count with one atomic (scores of one row share their high bits, so
    // per-lane atomics would serialise on a few bins)
    for (int base = 0; base < ncand; base += 32) {
      const int j = base + lane;
      const uint32_t x = j < ncand ? bits(j) : 0u;
      const bool in = j < ncand && (x & pmask) == prefix;
      const uint32_t digit = in ? ((x >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (in && (__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], (unsigned)__popc(peers));
    }
    __syncwarp();
    unsigned c[8];
    unsigned mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = hist[lane * 8 + e];
      mine += c[e];
    }
    // suffix sum over lanes (higher lanes hold higher digits)
    unsigned suf = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned other = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += other;
    }
    const unsigned above = suf - mine;  // keys with a digit above this lane's bins
    const bool owner = (above < (unsigned)k) && ((unsigned)k <= suf);
    const unsigned ob = __ballot_sync(0xffffffffu, owner);
    const int src = __ffs(ob) - 1;
    int digit = 0;
    unsigned count_above = 0;
    if (lane == src) {
      unsigned acc = above;
      for (int e = 7; e >= 0; --e) {
        if (acc + c[e] >= (unsigned)k) {
          digit = lane * 8 + e;
          break;
        }
        acc += c[e];
      }
      count_above = acc;
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    count_above = __shfl_sync(0xffffffffu, count_above, src);
    prefix |= (uint32_t)digit << shift;
    pmask |= 255u << shift;
    k -= (int)count_above;
    __syncwarp();
  }
  // prefix holds the n-th largest score; take every larger score and the k
  // lowest-index ties
  int written = 0, ties_seen = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int j = base + lane;
    const bool valid = j < ncand;
    const uint32_t x = valid ? bits(j) : 0u;
    const bool gt = valid && x > prefix;
    const bool eq = valid && x == prefix;
    const unsigned em = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && ties_seen + __popc(em & lt_mask) < k);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out(written + __popc(tm & lt_mask), j);
    written += __popc(tm);
    ties_seen += __popc(em);
  }
  for (int j = written + lane; j < n; j += 32) out(j, -1);
}

// Register path of the same selection for rows with at most 32 NI candidates
// (NI per lane; warp_topn_regs below picks the smallest NI that holds the
// row, so short rows cost proportionally less).  Every candidate j gets the 64-bit key (score key << 32) |
// (0xFFFFFFFF - j), so larger keys rank first and equal scores rank by lower
// index; keys are distinct.  The n-th largest of the 32 per-lane maxima is a
// lower bound T0 of the n-th largest key (n lanes hold a key >= it); the keys
// >= T0 (normally a few dozen) are ranked exactly in shared memory (`cand`,
// kCand words per warp) to find the n-th largest key K, and every key >= K is
// emitted in ascending block order.  Returns false, having written nothing,
// when more than kCand keys reach T0; the caller then uses warp_topn.
constexpr int kTopnCand = 64;

template <int NI, typename ScoreFn, typename OutFn>
__device__ __forceinline__ bool warp_topn_regs_n(ScoreFn score, int ncmp, int ncand, int n,
                                                 unsigned long long* cand, OutFn out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (ncand <= n) {
    for (int j = lane; j < n; j += 32) out(j, j < ncand ? j : -1);
    return true;
  }
  unsigned long long key[NI];
  unsigned long long lmax = 0;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int j = lane + 32 * i;
    const uint32_t b = j < ncmp ? score_key(score(j)) : kZeroScoreKey;
    key[i] = j < ncand ? (((unsigned long long)b << 32) | (0xFFFFFFFFu - (uint32_t)j)) : 0ull;
    lmax = key[i] > lmax ? key[i] : lmax;
  }
  // T0 = n-th largest lane maximum (at least n + 1 lanes hold candidates)
  int rank = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const unsigned long long other = __shfl_sync(0xffffffffu, lmax, o);
    rank += other > lmax;
  }
  const unsigned tb = __ballot_sync(0xffffffffu, rank == n - 1 && lmax != 0ull);
  const unsigned long long t0 = __shfl_sync(0xffffffffu, lmax, __ffs(tb) - 1);
  // gather the keys >= T0
  int count = 0;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const bool p = key[i] >= t0 && key[i] != 0ull;
    const unsigned m = __ballot_sync(0xffffffffu, p);
    const int pos = count + __popc(m & lt_mask);
    if (p && pos < kTopnCand) cand[pos] = key[i];
    count += __popc(m);
  }
  if (count > kTopnCand) return false;
  __syncwarp();
  // K = n-th largest gathered key
  unsigned long long kth = 0ull;
  bool have = false;
  for (int c = lane; c < count; c += 32) {
    const unsigned long long mine = cand[c];
    int r = 0;
    for (int d = 0; d < count; ++d) r += cand[d] > mine;
    if (r == n - 1) {
      kth = mine;
      have = true;
    }
  }
  const unsigned hb = __ballot_sync(0xffffffffu, have);
  kth = __shfl_sync(0xffffffffu, kth, __ffs(hb) - 1);
  __syncwarp();
  // every key >= K, in ascending block order
  int written = 0;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const bool take = key[i] >= kth && key[i] != 0ull;
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (take) out(written + __popc(m & lt_mask), lane + 32 * i);
    written += __popc(m);
  }
  return true;
}

// Rows of at most 1024 candidates: the register path sized to the row.
template <typename ScoreFn, typename OutFn>
__device__ __forceinline__ bool warp_topn_regs(ScoreFn score, int ncmp, int ncand, int n,
                                               unsigned long long* cand, OutFn out) {
  if (ncand <= 128) return warp_topn_regs_n<4>(score, ncmp, ncand, n, cand, out);
  if (ncand <= 256) return warp_topn_regs_n<8>(score, ncmp, ncand, n, cand, out);
  if (ncand <= 512) return warp_topn_regs_n<16>(score, ncmp, ncand, n, cand, out);
  return warp_topn_regs_n<32>(score, ncmp, ncand, n, cand, out);
}

// The same selection as warp_topn_regs for any number of candidates whose
// scores `score(j)` are cheap to re-read (shared memory): one pass finds each
// lane's largest key (lane = j % 32), T0 = the n-th largest lane maximum; a
// second pass gathers the keys >= T0 into `cand` and ranks them exactly; a
// third writes every key >= the n-th largest in ascending block order.
// Returns false, having written nothing, when more than kTopnCand keys reach
// T0 (the caller then uses warp_topn).
template <typename ScoreFn, typename OutFn>
__device__ __forceinline__ bool warp_topn_reread(ScoreFn score, int ncmp, int ncand, int n,
                                                 unsigned long long* cand, OutFn out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (ncand <= n) {
    for (int j = lane; j < n; j += 32) out(j, j < ncand ? j : -1);
    return true;
  }
  auto key = [&](int j) -> unsigned long long {
    const uint32_t b = j < ncmp ? score_key(score(j)) : kZeroScoreKey;
    return ((unsigned long long)b << 32) | (0xFFFFFFFFu - (uint32_t)j);
  };
  unsigned long long lmax = 0;
  for (int j = lane; j < ncand; j += 32) {
    const unsigned long long k = key(j);
    lmax = k > lmax ? k : lmax;
  }
  int rank = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const unsigned long long other = __shfl_sync(0xffffffffu, lmax, o);
    rank += other > lmax;
  }
  const unsigned tb = __ballot_sync(0xffffffffu, rank == n - 1 && lmax != 0ull);
  const unsigned long long t0 = __shfl_sync(0xffffffffu, lmax, __ffs(tb) - 1);
  int count = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int j = base + lane;
    const unsigned long long k = j < ncand ? key(j) : 0ull;
    const bool p = k >= t0 && k != 0ull;
    const unsigned m = __ballot_sync(0xffffffffu, p);
    const int pos = count + __popc(m & lt_mask);
    if (p && pos < kTopnCand) cand[pos] = k;
    count += __popc(m);
  }
  if (count > kTopnCand) return false;
  __syncwarp();
  unsigned long long kth = 0ull;
  bool have = false;
  for (int c = lane; c < count; c += 32) {
    const unsigned long long mine = cand[c];
    int r = 0;
    for (int e = 0; e < count; ++e) r += cand[e] > mine;
    if (r == n - 1) {
      kth = mine;
      have = true;
    }
  }
  const unsigned hb = __ballot_sync(0xffffffffu, have);
  kth = __shfl_sync(0xffffffffu, kth, __ffs(hb) - 1);
  __syncwarp();
  int written = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int j = base + lane;
    const unsigned long long k = j < ncand ? key(j) : 0ull;
    const bool take = k >= kth && k != 0ull;
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (take) out(written + __popc(m & lt_mask), j);
    written += __popc(m);
  }
  return true;
}


// The same selection by the 128 threads of a warpgroup (t = 0..127; `sync`
// is a barrier over exactly those threads) for rows whose scores `score(j)`
// are cheap to re-read: thread t takes the largest key of candidates t,
// t + 128, ...; T0 = the n-th largest of the 128 thread maxima (at least n
// keys reach it); the keys >= T0 are gathered into `cand` and ranked
// exactly, and each of the n largest writes itself at its position in
// ascending block order.  Scratch: `smax` 128 words, `cand` kTopnCand words,
// `ctl` 2 words, all shared.  Returns false (uniformly), having written
// nothing, when more than kTopnCand keys reach T0.
template <typename ScoreFn, typename OutFn, typename SyncFn>
__device__ __forceinline__ bool group_topn_128(ScoreFn score, int ncmp, int ncand, int n, int t,
                                               unsigned long long* smax,
                                               unsigned long long* cand,
                                               unsigned long long* ctl, SyncFn sync, OutFn out) {
  if (ncand <= n) {
    for (int j = t; j < n; j += 128) out(j, j < ncand ? j : -1);
    return true;
  }
  auto key = [&](int j) -> unsigned long long {
    const uint32_t b = j < ncmp ? score_key(score(j)) : kZeroScoreKey;
    return ((unsigned long long)b << 32) | (0xFFFFFFFFu - (uint32_t)j);
  };
  unsigned long long lmax = 0;
  for (int j = t; j < ncand; j += 128) {
    const unsigned long long k = key(j);
    lmax = k > lmax ? k : lmax;
  }
  smax[t] = lmax;
  if (t == 0) ctl[1] = 0;
  sync();
  // T0: the thread maxima are distinct keys (or 0 for a thread without
  // candidates); more than n threads hold one because ncand > n
  int rank = 0;
  for (int u = 0; u < 128; ++u) rank += smax[u] > lmax;
  if (lmax != 0ull && rank == n - 1) ctl[0] = lmax;
  sync();
  const unsigned long long t0 = ctl[0];
  for (int j = t; j < ncand; j += 128) {
    const unsigned long long k = key(j);
    if (k >= t0) {
      const unsigned long long pos = atomicAdd(ctl + 1, 1ull);
      if (pos < (unsigned long long)kTopnCand) cand[pos] = k;
    }
  }
  sync();
  const int count = (int)ctl[1];
  if (count > kTopnCand) return false;
  // the n-th largest gathered key
  unsigned long long mine = 0;
  if (t < count) {
    mine = cand[t];
    int r = 0;
    for (int e = 0; e < count; ++e) r += cand[e] > mine;
    if (r == n - 1) ctl[0] = mine;
  }
  sync();
  const unsigned long long kth = ctl[0];
  if (t < count && mine >= kth) {
    // position among the selected keys in ascending block order (a larger
    // key field below the score means a smaller block index)
    const uint32_t jm = 0xFFFFFFFFu - (uint32_t)(mine & 0xFFFFFFFFull);
    int pos = 0;
    for (int e = 0; e < count; ++e) {
      const unsigned long long o = cand[e];
      pos += (o >= kth) && ((0xFFFFFFFFu - (uint32_t)(o & 0xFFFFFFFFull)) < jm);
    }
    out(pos, (int)jm);
  }
  return true;
}

}  // namespace nsa
