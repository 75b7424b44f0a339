// Decode: the NSA forward pass (steps 1-7) for the newest token of each
// sequence of a batch whose keys and values sit in a dense KV cache (the
// config page separates prefill from decode in its benchmarking advice,
// section 5).
//
// A decode step reads every compressed block, the window and the selected
// blocks of each (sequence, KV group) once: an HBM-bound stream of about
// 1.3 MB per pair at the 64k shape.  It is cut into units of similar size so
// that every SM streams, with no unit waiting for another:
//   nsa_decode_compress_kernel  when the newest token completes a
//              compressed block (len >= l, (len - l) % d == 0), that block
//              is compressed from the cache (step 1) into the compressed
//              cache;
//   nsa_decode_a_kernel  one CTA per pair, the dependency the selected
//              keys wait for: all compressed keys through a six-stage ring,
//              S^T = Kc Q^T (keys on TMEM lanes, the group's heads on 16
//              columns), per-head log-sum-exp, the normalised probabilities
//              P^T (bf16, to the workspace), the block scores (step 3: the
//              sum over heads of p, summed over the compressed blocks
//              overlapping each selection block when l, d and l' differ)
//              and the top-n (step 4, one warp, to the workspace and
//              sel_idx);
//   nsa_decode_b_kernel  units of at most four 128-key chunks per pair:
//     cmp      O_cmp partial sums P Vc over a range of compressed blocks
//              (step 2, with the probabilities of kernel A);
//     window   a range of the w keys ending at t (step 6);
//     selected a range of the selected blocks (step 5; the incomplete
//              block holding t is loaded as the l' rows ending at t);
//              window and selected units leave a softmax partial (row
//              maximum, sum, unnormalised O);
//   the last unit of a pair to finish (an atomic counter per pair) merges
//   the partials and applies the gates (step 7):
//     out = g_cmp O_cmp + g_slc O_slc + g_win O_win.
// Both kernels: warp 0 = TMA producer, warp 1 = tcgen05.mma issuer,
// warps 2..5 = softmax / epilogue (thread = key lane of a chunk, or channel).
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "softmax_util.cuh"
#include "topn_util.cuh"

namespace nsa {
using namespace sm100;

namespace {

// ------------------------------------------------------------------ step 1 for decode
// Kc[blk, h, c] = sum_k W[h, c, k] * X[b, blk*d + k / D, h, k % D] for the
// block the newest token completed.  One warp per output channel at a time;
// lanes split the l*D inputs (coalesced rows of W) and reduce with shuffles.
__global__ void __launch_bounds__(256) nsa_decode_compress_kernel(DecodeArgs a) {
  const int b = blockIdx.x, h = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const int L = __ldg(a.seqlens + b);
  const int l = a.geo.l, dstride = a.geo.d, D = a.geo.D, H = a.geo.Hkv;
  if (L < l || L > a.cap || (L - l) % dstride != 0) return;
  const int blk = (L - l) / dstride;
  extern __shared__ float xs[];  // l*D inputs of the block
  const uint16_t* X =
      (is_v ? a.v_cache : a.k_cache) + ((size_t)b * a.cap + (size_t)blk * dstride) * H * D;
  const int K = l * D;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const int p = k / D, c = k - p * D;
    xs[k] = __uint_as_float((uint32_t)X[((size_t)p * H + h) * D + c] << 16);
  }
  __syncthreads();
  const float* W = (is_v ? a.w_v : a.w_k) + (size_t)h * D * K;
  uint16_t* out = (is_v ? a.v_cmp : a.k_cmp) + (((size_t)b * a.ccap + blk) * H + h) * D;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
  for (int c = warp; c < D; c += nwarps) {
    const float4* wrow = reinterpret_cast<const float4*>(W + (size_t)c * K);
    const float4* x4 = reinterpret_cast<const float4*>(xs);
    float acc = 0.f;
    for (int k = lane; k < K / 4; k += 32) {
      const float4 wv = __ldg(wrow + k), xv = x4[k];
      acc = fmaf(wv.x, xv.x, acc);
      acc = fmaf(wv.y, xv.y, acc);
      acc = fmaf(wv.z, xv.z, acc);
      acc = fmaf(wv.w, xv.w, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const __nv_bfloat16 bv = __float2bfloat16_rn(acc);
      out[c] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
}

// ------------------------------------------------------------------ shared pieces
constexpr int kDecThreads = 192;
// at most 8 compressed-value units (32 chunks of 128 blocks) and 4 selected
// units (16 chunks: top_n <= 32 blocks of 32 or 16 of 64) per pair, each of
// up to kUnitChunks chunks
constexpr int kMaxCmpUnits = (kDecodeMaxCmp / kChunk + kUnitChunks - 1) / kUnitChunks;
constexpr int kMaxSlcUnits = (16 + kUnitChunks - 1) / kUnitChunks;
constexpr int kMaxWinUnits = (8 + kUnitChunks - 1) / kUnitChunks;  // window <= 1024 keys
constexpr int kPChunkBytes = 4096;  // P^T of one chunk: 128 keys x 16 heads, bf16

// Per-(sequence, group) quantities of one decode query.
struct DecPair {
  int ok, b, g, L, t, C, ncc, nwc, nsc, ncand, cmp_row0, win_row0;
};

__device__ __forceinline__ DecPair dec_pair(const DecodeArgs& a, int pair) {
  DecPair p{};
  p.b = pair / a.geo.Hkv;
  p.g = pair % a.geo.Hkv;
  p.L = __ldg(a.seqlens + p.b);
  p.ok = p.L >= 1 && p.L <= a.cap;
  if (!p.ok) return p;
  p.t = p.L - 1;
  const int bpc = kChunk >> a.geo.lg_ls;
  p.nsc = (a.geo.n + bpc - 1) / bpc;
  if (a.select_only) {
    // routing candidates: the complete blocks before the own block t / l'
    p.C = p.t >> a.geo.lg_ls;
    p.ncc = (p.C + kChunk - 1) / kChunk;
    p.nwc = 0;
    p.ncand = p.C;
  } else {
    p.C = num_cmp_blocks(p.L, a.geo.l, a.geo.d);
    p.ncc = (p.C + kChunk - 1) / kChunk;
    const int wn = min(a.geo.w, p.L);
    p.nwc = (wn + kChunk - 1) / kChunk;
    p.ncand = p.t / a.geo.ls + 1;
  }
  p.cmp_row0 = p.C - kChunk * p.ncc;      // compressed chunks end at the last block
  p.win_row0 = p.t - kChunk * p.nwc + 1;  // window chunks end at t
  return p;
}

// First cache row of the selected block `blk` of l tokens as loaded (the
// incomplete block holding t is loaded as the l rows ending at t).
__device__ __forceinline__ int sel_row0(int blk, int l, int t) {
  return (blk * l + l - 1 > t) ? t - l + 1 : blk * l;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Sweep over `nchunks` S^T chunks of 16 columns starting at TMEM column
// `col` (lane = key): op(c, v[16]) for each chunk, the loads of four chunks
// in flight before one wait.
template <int kMaxChunks, typename Op>
__device__ __forceinline__ void sweep_chunks(uint32_t lane_addr, uint32_t col, int nchunks, Op op) {
  // not unrolled: a one-shot decode CTA pays for every instruction fetch, and
  // one group of four chunks is already a long straight run of code
#pragma unroll 1
  for (int c0 = 0; c0 < kMaxChunks; c0 += 4) {
    if (c0 >= nchunks) break;
    float v[64];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float u16[16];
      tmem_ld16(lane_addr + col + (c0 + cc) * 16, u16);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[cc * 16 + j] = u16[j];
    }
    tmem_ld_wait();
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      if (c0 + cc >= nchunks) break;
      float u16[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) u16[j] = v[cc * 16 + j];
      op(c0 + cc, u16);
    }
  }
}

// Stores 16 bf16 head values of key r into a P^T chunk laid out as the B
// operand of O^T += V^T P^T: [head half][key / 8][key % 8][8 heads].
__device__ __forceinline__ void store_pt(uint8_t* chunk, int r, const float (&p)[16]) {
  uint32_t pk[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
  uint8_t* base = chunk + (r >> 3) * 128 + (r & 7) * 16;
  *reinterpret_cast<uint4*>(base) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  *reinterpret_cast<uint4*>(base + 2048) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t tmem_col, uint32_t stage, uint32_t qs) {
  constexpr uint32_t id_qk = idesc_bf16(128, 16, false, false);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const uint32_t qoff = (ks >> 2) * 2048 + (ks & 3) * 32;   // Q^T halves: 16 rows
    const uint32_t soff = (ks >> 2) * 16384 + (ks & 3) * 32;  // chunk halves: 128 rows
    mma_bf16_ss(tmem_col, smem_desc(stage + soff, 16, 1024, kLayoutSw128),
                smem_desc(qs + qoff, 16, 1024, kLayoutSw128), id_qk, ks > 0);
  }
}

// O^T (D x 16 at tmem_col) (+)= V^T P^T for one 128-key chunk.
__device__ __forceinline__ void issue_pv(uint32_t tmem_col, uint32_t stage, uint32_t pchunk,
                                         bool accumulate) {
  constexpr uint32_t id_pv = idesc_bf16(128, 16, true, true);
#pragma unroll
  for (int ks = 0; ks < kChunk / 16; ++ks)
    mma_bf16_ss(tmem_col, smem_desc(stage + ks * 2048, 16384, 1024, kLayoutSw128),
                smem_desc(pchunk + ks * 256, 128, 2048, kLayoutNone), id_pv,
                (accumulate || ks > 0) ? 1u : 0u);
}

// Workspace records of one pair (fp32): compressed partial sums
// [ncv][G][D]; window and selected partials [nwu or nsl][G*D + 32] (O
// [G][D], then the row maximum m[16] and the sum[16] per head; every record
// 16-byte aligned).
constexpr int partial_floats(int G, int D) { return G * D + 32; }
struct PairRecs {
  float* win;
  float* cmp;
  float* slc;
  uint8_t* pt;
  int* sel;
};

__device__ __forceinline__ PairRecs pair_recs(const DecodeArgs& a, int pair) {
  const int G = a.geo.G, D = a.geo.D;
  PairRecs r;
  r.win = a.ws_win + (size_t)pair * a.nwu * partial_floats(G, D);
  r.cmp = a.ws_cmp + (size_t)pair * a.ncv_max * G * D;
  r.slc = a.ws_slc + (size_t)pair * a.nsl * partial_floats(G, D);
  r.pt = a.ws_pt + (size_t)pair * a.ncc_max * kPChunkBytes;
  r.sel = a.ws_sel + (size_t)pair * a.geo.n;
  return r;
}

// ------------------------------------------------------------------ kernel A
// The PV products read a ring stage as a 128-channel operand (two 64-channel
// halves 16 KB apart).  With D = 64 only the first half exists: the second
// feeds output channels that are never read, and the pad after the ring keeps
// that read of the last stage inside the CTA's shared memory.
template <int D>
constexpr int ring_pad() { return D == 64 ? 16384 : 0; }

template <int D>
struct DecALayout {
  static constexpr int kStages = 6;
  static constexpr int kChunkBytes = kChunk * D * 2;
  static constexpr int kQ = 0;                                   // 16 x D bf16 (4 KB max)
  static constexpr int kRing = 4096;
  static constexpr int kU = kRing + kStages * kChunkBytes;       // scores [kDecodeMaxCmp]
  static constexpr int kRed = kU + kDecodeMaxCmp * 4;            // float [2][64]
  static constexpr int kSel = kRed + 2 * 64 * 4;                 // int [64]
  static constexpr int kHist = kSel + 64 * 4;                    // unsigned [256]
  static constexpr int kCand = kHist + 256 * 4;                  // u64 [kTopnCand]
  static constexpr int kMax = kCand + kTopnCand * 8;             // u64 [128] + [2]
  static constexpr int kBars = kMax + 130 * 8;
  static constexpr int kEnd = kBars + 24 * 8;
  static constexpr int kSmem = kEnd + 1024;  // manual 1024-byte alignment
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kStages <= 6, "barrier arrays");
};

template <int D>
__global__ void __launch_bounds__(kDecThreads)
    nsa_decode_a_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ DecodeMaps maps) {
  using L = DecALayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* st_full = bars + 1;   // [kStages]
  uint64_t* st_empty = bars + 7;  // [kStages]
  uint64_t* s_full = bars + 13;
  uint64_t* fin = bars + 14;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  unsigned* hist = reinterpret_cast<unsigned*>(sm + L::kHist);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(sm + L::kCand);
  unsigned long long* smax = reinterpret_cast<unsigned long long*>(sm + L::kMax);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int pair = blockIdx.x;
  const DecPair P = dec_pair(a, pair);
  if (!P.ok) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDeviceBadInputCode);
    return;
  }
  const int nchunks = P.ncc;
  const PairRecs rec = pair_recs(a, pair);
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // TMEM: S^T of up to 32 chunks (16 columns each)
  const uint32_t ncols = nchunks <= 8 ? 128u : (nchunks <= 16 ? 256u : 512u);
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  int* status = a.status;
  const int G = a.geo.G, n = a.geo.n;
  const int b = P.b, g = P.g;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int sc = 0;
      bool ok = true;
      const int qrows = a.geo.Hq < 16 ? a.geo.Hq : 16;
      mbar_arrive_expect_tx(q_full, qrows * D * 2);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tma_load_3d(sm + L::kQ + h * 2048, &maps.q, q_full, h * 64, g * G, b);
      auto load_rows = [&](const CUtensorMap* map, int row0) {
        const int s = sc % L::kStages, u = sc / L::kStages;
        if (u > 0 && !mbar_wait(st_empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
        uint8_t* dst = sm + L::kRing + s * L::kChunkBytes;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_load_4d(dst + h * 16384, map, st_full + s, h * 64, g, row0, b);
        ++sc;
      };
      for (int c = 0; c < nchunks && ok; ++c) load_rows(&maps.kc, P.cmp_row0 + c * kChunk);
      volatile int never = 0;
      for (int s = 0; s < L::kStages && s < sc; ++s) {
        const int last = sc - 1 - ((sc - 1 - s) % L::kStages);
        mbar_wait(st_full + s, (last / L::kStages) & 1, &never, nullptr, kWaitCycles / 4);
      }
      mbar_wait(q_full, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int sc = 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, status, kWaitCycles);
      tc_fence_after();
      auto wait_stage = [&]() -> uint32_t {
        const int s = sc % L::kStages;
        if (!mbar_wait(st_full + s, (sc / L::kStages) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return 0;
        }
        tc_fence_after();
        return sbase + L::kRing + s * L::kChunkBytes;
      };
      for (int c = 0; c < nchunks && ok; ++c) {
        const uint32_t st = wait_stage();
        if (!ok) break;
        issue_qk<D>(tmem + c * 16, st, sbase + L::kQ);
        mma_commit(st_empty + (sc % L::kStages));
        ++sc;
      }
      mma_commit(s_full);
      mma_commit(fin);
      volatile int never = 0;
      mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // key lane of every chunk; channel in the epilogue
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const uint32_t colmask = (G >= 16) ? 0xFFFFu : ((1u << G) - 1u);
    // keys of this lane that take part (complete blocks), one bit per chunk
    uint32_t kok = 0;
    for (int c = 0; c < nchunks; ++c) kok |= (P.cmp_row0 + c * kChunk + r >= 0) ? (1u << c) : 0u;
    mbar_wait(s_full, 0, abort_flag, status, kWaitCycles);
    tc_fence_after();
    if (a.select_only) {
      // routing scores: the sum over the group's heads of q . mean key (one
      // sweep, no softmax), then the n - 1 best earlier blocks and the own one
      float* scores = reinterpret_cast<float*>(sm + L::kU);
      const bool live = !*abort_flag;
      sweep_chunks<32>(lane_addr, 0, nchunks, [&](int c, const float(&v)[16]) {
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h) s += ((colmask >> h) & 1u) ? v[h] : 0.f;
        if ((kok >> c) & 1u) scores[P.cmp_row0 + c * kChunk + r] = s;
      });
      named_bar_128<1>();
      int* gsel = a.sel ? a.sel + ((size_t)b * a.geo.Hkv + g) * n : nullptr;
      auto put = [&](int i, int j) {
        if (live) rec.sel[i] = j;
        if (gsel && live) gsel[i] = j;
      };
      auto sync = [&]() { named_bar_128<1>(); };
      auto plain = [&](int j) { return scores[j]; };
      const int C = P.C, m = n - 1;
      bool done = true;
      if (m > 0) done = group_topn_128(plain, C, C, m, r, smax, cand, smax + 128, sync, put);
      if (!done && warp == 2) warp_topn(plain, C, C, m, hist, put);
      sync();
      if (r == 0) {
        const int taken = C < m ? C : m;
        put(taken, P.t >> a.geo.lg_ls);
        for (int i = taken + 1; i < n; ++i) put(i, -1);
      }
    } else {
    // sweep 1: per-head maximum (log2 units)
    float mx[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
    sweep_chunks<32>(lane_addr, 0, nchunks, [&](int c, const float(&v)[16]) {
      if ((kok >> c) & 1u) {
#pragma unroll
        for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[h] * sl2);
      }
    });
    reduce16_across_128<1>(mx, red, q4, lane, true);
    float sm16[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) sm16[h] = 0.f;
    {
      // sweep 2: sums -> log2-sum-exp per head
      sweep_chunks<32>(lane_addr, 0, nchunks, [&](int c, const float(&v)[16]) {
        if ((kok >> c) & 1u) {
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if ((colmask >> h) & 1u) sm16[h] += ex2(v[h] * sl2 - mx[h]);
        }
      });
      reduce16_across_128<1>(sm16, red + 64, q4, lane, false);
      float lse[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) lse[h] = sm16[h] > 0.f ? mx[h] + __log2f(sm16[h]) : INFINITY;
      // sweep 3: normalised probabilities -> P^T (workspace) and block scores
      float* scores = reinterpret_cast<float*>(sm + L::kU);
      const bool live = !*abort_flag;
      sweep_chunks<32>(lane_addr, 0, nchunks, [&](int c, const float(&v)[16]) {
        const bool on = (kok >> c) & 1u;
        float p[16];
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          p[h] = (on && ((colmask >> h) & 1u)) ? ex2(v[h] * sl2 - lse[h]) : 0.f;
          s += p[h];
        }
        if (live) store_pt(rec.pt + (size_t)c * kPChunkBytes, r, p);
        const int j = P.cmp_row0 + c * kChunk + r;
        if (on) scores[j] = s;
      });
      named_bar_128<1>();
      // top-n (the four softmax warps; the workspace copy feeds the selected
      // units): the bound-and-rank selection over the shared-memory scores,
      // else (when too many keys tie at its bound) the radix select on one warp
      int* gsel = a.sel ? a.sel + ((size_t)b * a.geo.Hkv + g) * n : nullptr;
      auto put = [&](int i, int j) {
        if (live) rec.sel[i] = j;
        if (gsel && live) gsel[i] = j;
      };
      auto sync = [&]() { named_bar_128<1>(); };
      const int C = P.C;
      auto remapped = [&](int j) { return remap_score(a.geo, [&](int i) { return scores[i]; }, C, j); };
      auto plain = [&](int j) { return scores[j]; };
      const bool done = a.geo.remap
                            ? group_topn_128(remapped, P.ncand, P.ncand, n, r, smax, cand, smax + 128, sync, put)
                            : group_topn_128(plain, C, P.ncand, n, r, smax, cand, smax + 128, sync, put);
      if (!done && warp == 2) {
        if (a.geo.remap)
          warp_topn(remapped, P.ncand, P.ncand, n, hist, put);
        else
          warp_topn(plain, C, P.ncand, n, hist, put);
      }
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// ------------------------------------------------------------------ kernel B
template <int D>
struct DecBLayout {
  static constexpr int kStages = 2;
  static constexpr int kChunkBytes = kChunk * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kRing = 4096;
  static constexpr int kP = kRing + kStages * kChunkBytes + ring_pad<D>();  // 2 chunks of P^T
  static constexpr int kRed = kP + kUnitChunks * kPChunkBytes;  // float [2][64]
  static constexpr int kSel = kRed + 2 * 64 * 4;            // int [64]
  static constexpr int kFlag = kSel + 64 * 4;               // int
  static constexpr int kBars = kFlag + 16;
  static constexpr int kEnd = kBars + 16 * 8;
  static constexpr int kSmem = kEnd + 1024;
  // a PV operand spans 32 KB from the start of its stage
  static_assert(kRing + (kStages - 1) * kChunkBytes + 32768 <= kEnd, "PV operand inside smem");
  // two CTAs per SM (228 KB of shared memory, 1 KB reserved per CTA)
  static_assert(2 * (kSmem + 1024) <= 233472, "two CTAs per SM");
};

template <int D>
__global__ void __launch_bounds__(kDecThreads)
    nsa_decode_b_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ DecodeMaps maps) {
  using L = DecBLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* st_full = bars + 1;   // [3]
  uint64_t* st_empty = bars + 4;  // [3]
  uint64_t* pt_full = bars + 7;   // P^T chunks of a cmp unit
  uint64_t* s_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* o_done = bars + 10;
  uint64_t* fin = bars + 11;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  int* sel_s = reinterpret_cast<int*>(sm + L::kSel);
  int* last_flag = reinterpret_cast<int*>(sm + L::kFlag);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = a.ncv_max + a.nwu + a.nsl;
  const int pair = blockIdx.x / units, unit = blockIdx.x % units;
  const DecPair P = dec_pair(a, pair);
  if (!P.ok) return;  // kernel A has recorded the bad length
  // unit kinds: compressed values, window, selected blocks
  const bool is_cmp = unit < a.ncv_max;
  const bool is_win = !is_cmp && unit < a.ncv_max + a.nwu;
  const int u = is_cmp ? unit : (is_win ? unit - a.ncv_max : unit - a.ncv_max - a.nwu);
  // chunks [c_lo, c_hi) of the compressed blocks, the window or the selected keys
  const int total_chunks = is_cmp ? P.ncc : (is_win ? P.nwc : P.nsc);
  const int c_lo = min(kUnitChunks * u, total_chunks);
  const int c_hi = min(kUnitChunks * u + kUnitChunks, total_chunks);
  const int nch = c_hi - c_lo;
  const PairRecs rec = pair_recs(a, pair);
  // selection blocks of l' tokens
  const int G = a.geo.G, l = a.geo.ls, n = a.geo.n, lg_l = a.geo.lg_ls;
  const int bpc = kChunk >> lg_l;
  const int b = P.b, g = P.g, t = P.t;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(pt_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);  // S^T of four chunks at 0, 16, 32, 48; O^T at 64
    tmem_relinquish();
  }
  if (threadIdx.x < 64)
    sel_s[threadIdx.x] = (!is_cmp && !is_win && threadIdx.x < n) ? rec.sel[threadIdx.x] : -1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  int* status = a.status;

  if (nch > 0) {
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        int sc = 0;
        bool ok = true;
        auto acquire = [&]() -> uint8_t* {
          const int s = sc % L::kStages, uu = sc / L::kStages;
          if (uu > 0 && !mbar_wait(st_empty + s, (uu - 1) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            return nullptr;
          }
          mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
          return sm + L::kRing + s * L::kChunkBytes;
        };
        if (is_cmp) {
          mbar_arrive_expect_tx(pt_full, nch * kPChunkBytes);
          for (int c = 0; c < nch; ++c)
            bulk_load(sm + L::kP + c * kPChunkBytes, rec.pt + (size_t)(c_lo + c) * kPChunkBytes,
                      kPChunkBytes, pt_full);
          for (int c = c_lo; c < c_hi && ok; ++c) {
            uint8_t* dst = acquire();
            if (!dst) break;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(dst + h * 16384, &maps.vc, st_full + sc % L::kStages, h * 64, g,
                          P.cmp_row0 + c * kChunk, b);
            ++sc;
          }
        } else {
          const int qrows = a.geo.Hq < 16 ? a.geo.Hq : 16;
          mbar_arrive_expect_tx(q_full, qrows * D * 2);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sm + L::kQ + h * 2048, &maps.q, q_full, h * 64, g * G, b);
          for (int pass = 0; pass < 2 && ok; ++pass) {  // keys, then values
            for (int c = c_lo; c < c_hi && ok; ++c) {
              uint8_t* dst = acquire();
              if (!dst) break;
              const int s = sc % L::kStages;
              if (is_win) {  // 128 consecutive window rows ending at t
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                  tma_load_4d(dst + h * 16384, pass ? &maps.v_win : &maps.k_win, st_full + s, h * 64,
                              g, P.win_row0 + c * kChunk, b);
                ++sc;
                continue;
              }
              for (int sub = 0; sub < bpc; ++sub) {
                const int bs = c * bpc + sub;
                const int blk = bs < n ? sel_s[bs] : -1;
                const int row = blk >= 0 ? sel_row0(blk, l, t) : -(1 << 24);
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                  tma_load_4d(dst + h * 16384 + sub * l * 128, pass ? &maps.v_blk : &maps.k_blk,
                              st_full + s, h * 64, g, row, b);
              }
              ++sc;
            }
          }
        }
        volatile int never = 0;
        for (int s = 0; s < L::kStages && s < sc; ++s) {
          const int last = sc - 1 - ((sc - 1 - s) % L::kStages);
          mbar_wait(st_full + s, (last / L::kStages) & 1, &never, nullptr, kWaitCycles / 4);
        }
        if (is_cmp) mbar_wait(pt_full, 0, &never, nullptr, kWaitCycles / 4);
        else mbar_wait(q_full, 0, &never, nullptr, kWaitCycles / 4);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        int sc = 0;
        bool ok = true;
        auto wait_stage = [&]() -> uint32_t {
          const int s = sc % L::kStages;
          if (!mbar_wait(st_full + s, (sc / L::kStages) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            return 0;
          }
          tc_fence_after();
          return sbase + L::kRing + s * L::kChunkBytes;
        };
        if (is_cmp) {
          ok = mbar_wait(pt_full, 0, abort_flag, status, kWaitCycles);
          for (int c = 0; c < nch && ok; ++c) {
            const uint32_t st = wait_stage();
            if (!ok) break;
            issue_pv(tmem + 64, st, sbase + L::kP + c * kPChunkBytes, c > 0);
            mma_commit(st_empty + (sc % L::kStages));
            ++sc;
          }
        } else {
          ok = mbar_wait(q_full, 0, abort_flag, status, kWaitCycles);
          tc_fence_after();
          for (int c = 0; c < nch && ok; ++c) {
            const uint32_t st = wait_stage();
            if (!ok) break;
            issue_qk<D>(tmem + c * 16, st, sbase + L::kQ);
            mma_commit(st_empty + (sc % L::kStages));
            ++sc;
          }
          mma_commit(s_full);
          if (ok && mbar_wait(p_full, 0, abort_flag, status, kWaitCycles)) {
            tc_fence_after();
            for (int c = 0; c < nch && ok; ++c) {
              const uint32_t st = wait_stage();
              if (!ok) break;
              issue_pv(tmem + 64, st, sbase + L::kP + c * kPChunkBytes, c > 0);
              mma_commit(st_empty + (sc % L::kStages));
              ++sc;
            }
          }
        }
        mma_commit(o_done);
        mma_commit(fin);
        volatile int never = 0;
        mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
      }
    } else {
      // ---------------------------------------------------------- softmax / partial
      const int q4 = warp & 3;
      const int r = q4 * 32 + lane;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
      const float sl2 = a.geo.scale_log2;
      const uint32_t colmask = (G >= 16) ? 0xFFFFu : ((1u << G) - 1u);
      float mx[16], sm16[16];
      if (!is_cmp) {
        // keys of this lane that take part, per chunk: window keys from
        // max(0, t - w + 1), or visible keys of the selected blocks
        uint32_t kok = 0;
        if (is_win) {
          const int lo = max(0, t - a.geo.w + 1);
          for (int c = 0; c < nch; ++c)
            kok |= (P.win_row0 + (c_lo + c) * kChunk + r >= lo) ? (1u << c) : 0u;
        } else {
          const int key_in_blk = r & (l - 1), slot_in_chunk = r >> lg_l;
          for (int c = 0; c < nch; ++c) {
            const int bs = (c_lo + c) * bpc + slot_in_chunk;
            const int blk = bs < n ? sel_s[bs] : -1;
            kok |= (blk >= 0 && sel_row0(blk, l, t) + key_in_blk >= blk * l) ? (1u << c) : 0u;
          }
        }
        mbar_wait(s_full, 0, abort_flag, status, kWaitCycles);
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
        sweep_chunks<kUnitChunks>(lane_addr, 0, nch, [&](int c, const float(&v)[16]) {
          if ((kok >> c) & 1u) {
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[h] * sl2);
          }
        });
        reduce16_across_128<1>(mx, red, q4, lane, true);
#pragma unroll
        for (int h = 0; h < 16; ++h) sm16[h] = 0.f;
        sweep_chunks<kUnitChunks>(lane_addr, 0, nch, [&](int c, const float(&v)[16]) {
          const bool on = (kok >> c) & 1u;
          float p[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            p[h] = (on && ((colmask >> h) & 1u)) ? ex2(v[h] * sl2 - mx[h]) : 0.f;
            sm16[h] += p[h];
          }
          store_pt(sm + L::kP + c * kPChunkBytes, r, p);
        });
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        reduce16_across_128<1>(sm16, red + 64, q4, lane, false);
      }
      mbar_wait(o_done, 0, abort_flag, status, kWaitCycles);
      tc_fence_after();
      float o[16];
      tmem_ld16(lane_addr + 64, o);
      tmem_ld_wait();
      if (r < D && !*abort_flag) {
        if (is_cmp) {
          float* dst = rec.cmp + (size_t)u * G * D;
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            if (h >= G) break;
            dst[h * D + r] = o[h];
          }
        } else {
          float* dst = (is_win ? rec.win : rec.slc) + (size_t)u * partial_floats(G, D);
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            if (h >= G) break;
            dst[h * D + r] = o[h];
          }
          if (r < G) {
            float mv = 0.f, lv = 0.f;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
              mv = (h == r) ? mx[h] : mv;
              lv = (h == r) ? sm16[h] : lv;
            }
            dst[G * D + r] = mv;
            dst[G * D + 16 + r] = lv;
          }
        }
      }
    }
  } else if (warp >= 2 && !is_cmp) {
    // a selected unit with no chunk: an empty partial
    const int r = threadIdx.x - 64;
    float* dst = (is_win ? rec.win : rec.slc) + (size_t)u * partial_floats(G, D);
    if (r < D)
      for (int h = 0; h < G; ++h) dst[h * D + r] = 0.f;
    if (r < G) {
      dst[G * D + r] = -INFINITY;
      dst[G * D + 16 + r] = 0.f;
    }
  }
  // ---- the last unit of the pair merges the partials (step 7)
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int done = atomicAdd(a.counters + pair, 1);
    *last_flag = done == units - 1;
  }
  __syncthreads();
  if (*last_flag) {
    __threadfence();
    // per-head statistics of the selected partials and the gates, staged in
    // the (now idle) P^T region; then every (head, 4 channels) item issues
    // all of its partial loads before combining them
    float* ml = reinterpret_cast<float*>(sm + L::kP);  // selected [nsl][m[16], sum[16]]
    float* wml = ml + kMaxSlcUnits * 32;                // window [nwu][m[16], sum[16]]
    float* gt = wml + kMaxWinUnits * 32;                // [G][3]
    const int Hq = a.geo.Hq, PF = partial_floats(G, D);
    for (int i = threadIdx.x; i < a.nsl * 32; i += blockDim.x)
      ml[i] = __ldcg(rec.slc + (size_t)(i >> 5) * PF + G * D + (i & 31));
    for (int i = threadIdx.x; i < a.nwu * 32; i += blockDim.x)
      wml[i] = __ldcg(rec.win + (size_t)(i >> 5) * PF + G * D + (i & 31));
    for (int i = threadIdx.x; i < G * 3; i += blockDim.x)
      gt[i] = a.select_only ? ((i % 3) == 1 ? 1.f : 0.f)  // the selected branch alone
                            : __ldg(a.gates + ((size_t)b * Hq + g * G) * 3 + i);
    __syncthreads();
    const int ncv = a.select_only ? 0 : (P.ncc + kUnitChunks - 1) / kUnitChunks;
    for (int item = threadIdx.x; item < G * (D / 4); item += blockDim.x) {
      const int h = item / (D / 4), c4 = (item - h * (D / 4)) * 4;
      float4 vs[kMaxSlcUnits], vw[kMaxWinUnits], vc[kMaxCmpUnits];
#pragma unroll
      for (int s2 = 0; s2 < kMaxSlcUnits; ++s2)
        if (s2 < a.nsl)
          vs[s2] = __ldcg(reinterpret_cast<const float4*>(rec.slc + (size_t)s2 * PF + h * D + c4));
#pragma unroll
      for (int s2 = 0; s2 < kMaxWinUnits; ++s2)
        if (s2 < a.nwu)
          vw[s2] = __ldcg(reinterpret_cast<const float4*>(rec.win + (size_t)s2 * PF + h * D + c4));
#pragma unroll
      for (int u2 = 0; u2 < kMaxCmpUnits; ++u2)
        if (u2 < ncv)
          vc[u2] = __ldcg(reinterpret_cast<const float4*>(rec.cmp + ((size_t)u2 * G + h) * D + c4));
      // softmax partials (row maximum m, sum, unnormalised O) -> normalised O
      auto merge = [&](const float* mlv, const auto& v, int units_of) {
        constexpr int kMax = sizeof(v) / sizeof(float4);  // unrolled: v stays in registers
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kMax; ++s2)
          if (s2 < units_of) M = fmaxf(M, mlv[s2 * 32 + h]);
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float ls = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kMax; ++s2) {
          if (s2 >= units_of) break;
          const float ms = mlv[s2 * 32 + h];
          const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : ex2(ms - M);
          ls += mlv[s2 * 32 + 16 + h] * f;
          o.x += v[s2].x * f;
          o.y += v[s2].y * f;
          o.z += v[s2].z * f;
          o.w += v[s2].w * f;
        }
        const float inv = ls > 0.f ? 1.f / ls : 0.f;
        return make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      };
      const float4 os = merge(ml, vs, a.nsl);
      const float4 ow = merge(wml, vw, a.nwu);
      float4 oc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u2 = 0; u2 < kMaxCmpUnits; ++u2) {
        if (u2 >= ncv) break;
        oc.x += vc[u2].x;
        oc.y += vc[u2].y;
        oc.z += vc[u2].z;
        oc.w += vc[u2].w;
      }
      const float g0 = gt[h * 3 + 0], g1 = gt[h * 3 + 1], g2 = gt[h * 3 + 2];
      const float e[4] = {g0 * oc.x + g1 * os.x + g2 * ow.x, g0 * oc.y + g1 * os.y + g2 * ow.y,
                          g0 * oc.z + g1 * os.z + g2 * ow.z, g0 * oc.w + g1 * os.w + g2 * ow.w};
      const size_t oi = ((size_t)b * Hq + g * G + h) * D + c4;
      if (a.geo.out_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + oi) = make_float4(e[0], e[1], e[2], e[3]);
      } else {
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + oi) =
            make_uint2(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]));
      }
    }
    if (threadIdx.x == 0) a.counters[pair] = 0;
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes, bool (&configured)[64]) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_decode_a_t(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  static bool conf[64] = {};
  cudaError_t e = set_smem(nsa_decode_a_kernel<D>, DecALayout<D>::kSmem, conf);
  if (e != cudaSuccess) return e;
  nsa_decode_a_kernel<D><<<a.batch * a.geo.Hkv, kDecThreads, DecALayout<D>::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_b_t(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  static bool conf[64] = {};
  cudaError_t e = set_smem(nsa_decode_b_kernel<D>, DecBLayout<D>::kSmem, conf);
  if (e != cudaSuccess) return e;
  const int grid = a.batch * a.geo.Hkv * (a.ncv_max + a.nwu + a.nsl);
  nsa_decode_b_kernel<D><<<grid, kDecThreads, DecBLayout<D>::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_compress(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)a.geo.l * a.geo.D * sizeof(float);
  static bool configured[64] = {};
  cudaError_t e = set_smem(nsa_decode_compress_kernel, 64 * 128 * 4, configured);
  if (e != cudaSuccess) return e;
  nsa_decode_compress_kernel<<<dim3(a.batch, a.geo.Hkv, 2), 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_a(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  return a.geo.D == 128 ? launch_decode_a_t<128>(a, m, s) : launch_decode_a_t<64>(a, m, s);
}

cudaError_t launch_decode_b(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  return a.geo.D == 128 ? launch_decode_b_t<128>(a, m, s) : launch_decode_b_t<64>(a, m, s);
}

}  // namespace nsa
