// Decode: the NSA forward pass (steps 1-7) for the newest token of each
// sequence of a batch whose keys and values sit in a dense KV cache (the
// config page separates prefill from decode in its benchmarking advice,
// section 5).
//
// nsa_decode_compress_kernel: when the newest token completes a block
// (len % l == 0), that block is compressed from the cache (step 1) and
// written into the compressed cache; all other blocks were compressed before.
//
// nsa_decode_kernel: one CTA per (sequence, KV group), the group's G heads
// sharing every load.  All products are swap-AB tcgen05 MMAs with 128 keys on
// the TMEM lanes and the heads on 16 columns (S^T = K Q^T, O^T += V^T P^T):
//   compressed all complete blocks (chunks end at the last one), two-sweep
//             softmax, O_cmp, and a third sweep for the block scores
//             S_j = sum over heads of the normalised probabilities;
//   top-n     one warp selects n blocks from the scores in shared memory
//             (the window's keys and values stream in meanwhile);
//   window    the w tokens ending at t (chunks end at t, so no cache row past
//             the sequence is read), two-sweep softmax, O_win;
//   selected  the chosen blocks (the incomplete block is loaded as the l rows
//             ending at t), two-sweep softmax, O_slc;
//   epilogue  out = g_cmp O_cmp + g_slc O_slc + g_win O_win, lane = channel.
// Warp roles: 0 = TMA producer, 1 = MMA issuer, 2..5 = softmax / top-n /
// epilogue.  Memory per (sequence, group) at the 64k shape: 512 KB of
// compressed KV, 512 KB of selected blocks and 256 KB of window, streamed
// through a 4-stage ring of 32 KB chunks.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "softmax_util.cuh"
#include "topn_util.cuh"

namespace nsa {
using namespace sm100;

namespace {

// ------------------------------------------------------------------ step 1 for decode
// Kc[blk, h, c] = sum_k W[h, c, k] * X[b, blk*l + k / D, h, k % D] for the
// block the newest token completed.  One warp per 16 output channels; lanes
// split the l*D inputs (coalesced rows of W) and reduce with shuffles.
__global__ void __launch_bounds__(256) nsa_decode_compress_kernel(DecodeArgs a) {
  const int b = blockIdx.x, h = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const int L = __ldg(a.seqlens + b);
  const int l = a.geo.l, D = a.geo.D, H = a.geo.Hkv;
  if (L < l || L > a.cap || (L % l) != 0) return;
  const int blk = L / l - 1;
  extern __shared__ float xs[];  // l*D inputs of the block
  const uint16_t* X = (is_v ? a.v_cache : a.k_cache) + ((size_t)b * a.cap + (size_t)blk * l) * H * D;
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
    const float* wrow = W + (size_t)c * K;
    float acc = 0.f;
    for (int k = lane; k < K; k += 32) acc = fmaf(__ldg(wrow + k), xs[k], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const __nv_bfloat16 bv = __float2bfloat16_rn(acc);
      out[c] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
}

// ------------------------------------------------------------------ fused decode
template <int D>
struct DecLayout {
  static constexpr int kStages = 4;
  static constexpr int kQBytes = 16 * D * 2;          // 16 head rows
  static constexpr int kChunkBytes = kChunk * D * 2;  // 128 keys
  static constexpr int kPBytes = 8 * 4096;            // 8 chunks of P^T (128 keys x 16 heads)
  static constexpr int kQ = 0;
  static constexpr int kRing = 4096;                  // Q needs at most 4 KB
  static constexpr int kP = kRing + kStages * kChunkBytes;  // 2 buffers
  static constexpr int kScores = kP + 2 * kPBytes;          // float[1024]
  static constexpr int kRed = kScores + kDecodeMaxCmp * 4;  // float[2][64]
  static constexpr int kSel = kRed + 2 * 64 * 4;            // int[64]
  static constexpr int kHist = kSel + 64 * 4;               // unsigned[256]
  static constexpr int kBars = kHist + 256 * 4;
  static constexpr int kEnd = kBars + 32 * 8;
  static constexpr int kSmem = kEnd + 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr uint32_t kColSW = 0, kColSC = 128, kColSS = 256;
constexpr uint32_t kColOW = 384, kColOC = 400, kColOS = 416;

struct DecItem {
  int ok, b, g, L, t, C, nwc, ncc, nsc, ncand;
};

__device__ __forceinline__ DecItem dec_item(const DecodeArgs& a) {
  DecItem it{};
  it.b = blockIdx.x / a.geo.Hkv;
  it.g = blockIdx.x % a.geo.Hkv;
  it.L = __ldg(a.seqlens + it.b);
  it.ok = it.L >= 1 && it.L <= a.cap && it.L / a.geo.l <= kDecodeMaxCmp;
  if (!it.ok) return it;
  it.t = it.L - 1;
  it.C = it.L / a.geo.l;
  const int wn = min(a.geo.w, it.L);
  it.nwc = (wn + kChunk - 1) / kChunk;
  it.ncc = (it.C + kChunk - 1) / kChunk;
  const int bpc = kChunk >> a.geo.lg_l;
  it.nsc = (a.geo.n + bpc - 1) / bpc;
  it.ncand = it.t / a.geo.l + 1;
  return it;
}

// First cache row of the selected block `blk` as loaded (the incomplete block
// holding t is loaded as the l rows ending at t).
__device__ __forceinline__ int sel_row0(int blk, int l, int t) {
  return (blk * l + l - 1 > t) ? t - l + 1 : blk * l;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    nsa_decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ DecodeMaps maps) {
  using L = DecLayout<D>;
  constexpr int KSTEPS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* st_full = bars + 1;   // [4]
  uint64_t* st_empty = bars + 5;  // [4]
  uint64_t* sW_full = bars + 9;
  uint64_t* sC_full = bars + 10;
  uint64_t* sS_full = bars + 11;
  uint64_t* pW_full = bars + 12;
  uint64_t* pC_full = bars + 13;
  uint64_t* pS_full = bars + 14;
  uint64_t* pW_empty = bars + 15;
  uint64_t* idx_ready = bars + 16;
  uint64_t* o_done = bars + 17;
  uint64_t* fin = bars + 18;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 20);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  float* scores = reinterpret_cast<float*>(sm + L::kScores);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  int* sel_s = reinterpret_cast<int*>(sm + L::kSel);
  unsigned* hist = reinterpret_cast<unsigned*>(sm + L::kHist);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const DecItem it = dec_item(a);
  if (!it.ok) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDeviceBadInputCode);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(sW_full, 1);
    mbar_init(sC_full, 1);
    mbar_init(sS_full, 1);
    mbar_init(pW_full, 4);
    mbar_init(pC_full, 4);
    mbar_init(pS_full, 4);
    mbar_init(pW_empty, 1);
    mbar_init(idx_ready, 1);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  int* status = a.status;
  const int G = a.geo.G, l = a.geo.l, n = a.geo.n, lg_l = a.geo.lg_l;
  const int bpc = kChunk >> lg_l;
  const int t = it.t, b = it.b, g = it.g;
  const int win_row0 = t - kChunk * it.nwc + 1;  // first row of window chunk 0
  const int cmp_row0 = it.C - kChunk * it.ncc;   // first row of compressed chunk 0

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int sc = 0;
      bool ok = true;
      auto acquire = [&]() -> uint8_t* {
        const int s = sc % L::kStages, u = sc / L::kStages;
        if (u > 0 && !mbar_wait(st_empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return nullptr;
        }
        mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
        return sm + L::kRing + s * L::kChunkBytes;
      };
      // 128 rows of a [rows, Hkv, D] cache slab starting at row0 (rows < 0 read 0)
      auto load_rows = [&](const CUtensorMap* map, int row0) {
        uint8_t* dst = acquire();
        if (!dst) return;
        const int s = sc % L::kStages;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_load_4d(dst + h * 16384, map, st_full + s, h * 64, g, row0, b);
        ++sc;
      };
      auto load_sel = [&](bool is_v) {
        for (int c = 0; c < it.nsc && ok; ++c) {
          uint8_t* dst = acquire();
          if (!dst) return;
          const int s = sc % L::kStages;
          for (int sub = 0; sub < bpc; ++sub) {
            const int bs = c * bpc + sub;
            const int blk = bs < n ? sel_s[bs] : -1;
            const int row = blk >= 0 ? sel_row0(blk, l, t) : -(1 << 24);
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(dst + h * 16384 + sub * l * 128, is_v ? &maps.v_blk : &maps.k_blk,
                          st_full + s, h * 64, g, row, b);
          }
          ++sc;
        }
      };
      // 16 head rows per 64-channel half (fewer when Hq < 16; the rows the box
      // leaves untouched only feed result columns that are never read)
      const int qrows = a.geo.Hq < 16 ? a.geo.Hq : 16;
      mbar_arrive_expect_tx(q_full, qrows * D * 2);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tma_load_3d(sm + L::kQ + h * 2048, &maps.q, q_full, h * 64, g * G, b);
      // compressed keys first: the block scores (and the top-n that the
      // selected loads wait for) are computed while the rest streams in
      for (int c = 0; c < it.ncc && ok; ++c) load_rows(&maps.kc, cmp_row0 + c * kChunk);
      for (int c = 0; c < it.nwc && ok; ++c) load_rows(&maps.k_win, win_row0 + c * kChunk);
      for (int c = 0; c < it.ncc && ok; ++c) load_rows(&maps.vc, cmp_row0 + c * kChunk);
      for (int c = 0; c < it.nwc && ok; ++c) load_rows(&maps.v_win, win_row0 + c * kChunk);
      if (ok && mbar_wait(idx_ready, 0, abort_flag, status, kWaitCycles)) {
        load_sel(false);
        if (ok) load_sel(true);
      }
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
      constexpr uint32_t id_qk = idesc_bf16(128, 16, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, 16, true, true);
      const uint32_t Qs = sbase + L::kQ, Ps = sbase + L::kP;
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
      auto release_stage = [&]() {
        mma_commit(st_empty + (sc % L::kStages));
        ++sc;
      };
      auto qk = [&](int nchunks, uint32_t col) {
        for (int c = 0; c < nchunks && ok; ++c) {
          const uint32_t st = wait_stage();
          if (!ok) return;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            const uint32_t qoff = (ks >> 2) * 2048 + (ks & 3) * 32;   // Q^T halves: 16 rows
            const uint32_t soff = (ks >> 2) * 16384 + (ks & 3) * 32;  // chunk halves: 128 rows
            mma_bf16_ss(tmem + col + c * 16, smem_desc(st + soff, 16, 1024, kLayoutSw128),
                        smem_desc(Qs + qoff, 16, 1024, kLayoutSw128), id_qk, ks > 0);
          }
          release_stage();
        }
      };
      auto pv = [&](int nchunks, uint32_t pbuf, uint32_t col) {
        for (int c = 0; c < nchunks && ok; ++c) {
          const uint32_t st = wait_stage();
          if (!ok) return;
#pragma unroll
          for (int ks = 0; ks < kChunk / 16; ++ks)
            mma_bf16_ss(tmem + col, smem_desc(st + ks * 2048, 16384, 1024, kLayoutSw128),
                        smem_desc(pbuf + c * 4096 + ks * 256, 128, 2048, kLayoutNone), id_pv,
                        (c > 0 || ks > 0) ? 1u : 0u);
          release_stage();
        }
      };
      if (ok && it.ncc > 0) {
        qk(it.ncc, kColSC);
        mma_commit(sC_full);
      }
      if (ok) {
        qk(it.nwc, kColSW);
        mma_commit(sW_full);
      }
      if (ok && it.ncc > 0 && mbar_wait(pC_full, 0, abort_flag, status, kWaitCycles)) {
        tc_fence_after();
        pv(it.ncc, Ps + L::kPBytes, kColOC);
      }
      if (ok && mbar_wait(pW_full, 0, abort_flag, status, kWaitCycles)) {
        tc_fence_after();
        pv(it.nwc, Ps, kColOW);
        mma_commit(pW_empty);
      }
      if (ok) {
        qk(it.nsc, kColSS);
        mma_commit(sS_full);
      }
      if (ok && mbar_wait(pS_full, 0, abort_flag, status, kWaitCycles)) {
        tc_fence_after();
        pv(it.nsc, Ps, kColOS);
      }
      mma_commit(o_done);
      mma_commit(fin);
      volatile int never = 0;
      mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------ softmax / top-n / epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // key lane of every chunk; channel in the epilogue
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const uint32_t colmask = (G >= 16) ? 0xFFFFu : ((1u << G) - 1u);
    // Two-sweep softmax over the S^T chunks at `col` (keys on lanes, heads on
    // columns): writes unnormalised P^T into `pbuf` and returns 1/sum per head.
    auto softmax = [&](uint32_t col, int nchunks, const bool (&kok)[8], uint32_t pbuf,
                       float (&inv)[16]) {
      float mx[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < 8; c0 += 4) {
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
        for (int cc = 0; cc < 4; ++cc)
          if (c0 + cc < nchunks && kok[c0 + cc]) {
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[cc * 16 + h] * sl2);
          }
      }
      reduce16_across_128<1>(mx, red, q4, lane, true);
      float sm16[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) sm16[h] = 0.f;
      const uint32_t pb = pbuf + (r >> 3) * 128 + (r & 7) * 16;
#pragma unroll
      for (int c0 = 0; c0 < 8; c0 += 4) {
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
          const int c = c0 + cc;
          if (c >= nchunks) break;
          float p[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            p[h] = (kok[c] && ((colmask >> h) & 1u)) ? ex2(v[cc * 16 + h] * sl2 - mx[h]) : 0.f;
            sm16[h] += p[h];
          }
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
          st_shared_v4(pb + c * 4096, pk[0], pk[1], pk[2], pk[3]);
          st_shared_v4(pb + c * 4096 + 2048, pk[4], pk[5], pk[6], pk[7]);
        }
      }
      fence_async_smem();
      reduce16_across_128<1>(sm16, red + 64, q4, lane, false);
#pragma unroll
      for (int h = 0; h < 16; ++h) inv[h] = (((colmask >> h) & 1u) && sm16[h] > 0.f) ? 1.f / sm16[h] : 0.f;
    };
    const uint32_t P0 = sbase + L::kP, P1 = P0 + L::kPBytes;
    float inv_w[16], inv_c[16], inv_s[16];
    // ---- compressed branch and block scores
#pragma unroll
    for (int h = 0; h < 16; ++h) inv_c[h] = 0.f;
    if (it.ncc > 0) {
      bool kok[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) kok[c] = c < it.ncc && cmp_row0 + c * kChunk + r >= 0;
      mbar_wait(sC_full, 0, abort_flag, status, kWaitCycles);
      tc_fence_after();
      // sweep 1: per-head maximum (kept for the scores of sweep 3)
      float mx[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
      {
#pragma unroll
        for (int c0 = 0; c0 < 8; c0 += 4) {
          if (c0 >= it.ncc) break;
          float v[64];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float u16[16];
            tmem_ld16(lane_addr + kColSC + (c0 + cc) * 16, u16);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[cc * 16 + j] = u16[j];
          }
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            if (c0 + cc < it.ncc && kok[c0 + cc]) {
#pragma unroll
              for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[cc * 16 + h] * sl2);
            }
        }
      }
      reduce16_across_128<1>(mx, red, q4, lane, true);
      // sweep 2: P^T and sums; sweep 3: normalised probabilities summed over heads
      float sm16[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) sm16[h] = 0.f;
      const uint32_t pb = P1 + (r >> 3) * 128 + (r & 7) * 16;
      for (int c = 0; c < it.ncc; ++c) {
        float v[16];
        tmem_ld16(lane_addr + kColSC + c * 16, v);
        tmem_ld_wait();
        float p[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          p[h] = (kok[c] && ((colmask >> h) & 1u)) ? ex2(v[h] * sl2 - mx[h]) : 0.f;
          sm16[h] += p[h];
        }
        uint32_t pk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
        st_shared_v4(pb + c * 4096, pk[0], pk[1], pk[2], pk[3]);
        st_shared_v4(pb + c * 4096 + 2048, pk[4], pk[5], pk[6], pk[7]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pC_full);
      reduce16_across_128<1>(sm16, red + 64, q4, lane, false);
      // log2 of each head's normaliser: p_norm = 2^(s*sl2 - mx - log2(sum))
      float lnorm[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        inv_c[h] = (((colmask >> h) & 1u) && sm16[h] > 0.f) ? 1.f / sm16[h] : 0.f;
        lnorm[h] = sm16[h] > 0.f ? mx[h] + __log2f(sm16[h]) : INFINITY;
      }
      for (int c = 0; c < it.ncc; ++c) {
        float v[16];
        tmem_ld16(lane_addr + kColSC + c * 16, v);
        tmem_ld_wait();
        const int j = cmp_row0 + c * kChunk + r;
        if (kok[c]) {
          float s = 0.f;
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if ((colmask >> h) & 1u) s += ex2(v[h] * sl2 - lnorm[h]);
          scores[j] = s;
        }
      }
    }
    // ---- top-n (one warp), indices to shared memory, global output and the producer
    named_bar_128<1>();
    if (warp == 2) {
      int* gsel = a.sel ? a.sel + ((size_t)b * a.geo.Hkv + g) * n : nullptr;
      warp_topn([&](int j) { return scores[j]; }, it.C, it.ncand, n, hist, [&](int i, int j) {
        sel_s[i] = j;
        if (gsel) gsel[i] = j;
      });
      __syncwarp();
      if (lane == 0) mbar_arrive(idx_ready);
    }
    named_bar_128<1>();
    // ---- window
    {
      bool kok[8];
      const int lo = max(0, t - a.geo.w + 1);
#pragma unroll
      for (int c = 0; c < 8; ++c) kok[c] = c < it.nwc && win_row0 + c * kChunk + r >= lo;
      mbar_wait(sW_full, 0, abort_flag, status, kWaitCycles);
      tc_fence_after();
      softmax(kColSW, it.nwc, kok, P0, inv_w);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pW_full);
    }
    // ---- selected branch
    {
      bool kok[8];
      const int key_in_blk = r & (l - 1), slot_in_chunk = r >> lg_l;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int bs = c * bpc + slot_in_chunk;
        const int blk = (c < it.nsc && bs < n) ? sel_s[bs] : -1;
        kok[c] = blk >= 0 && sel_row0(blk, l, t) + key_in_blk >= blk * l;
      }
      mbar_wait(sS_full, 0, abort_flag, status, kWaitCycles);
      mbar_wait(pW_empty, 0, abort_flag, status, kWaitCycles);
      tc_fence_after();
      softmax(kColSS, it.nsc, kok, P0, inv_s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pS_full);
    }
    // ---- epilogue: lane = channel
    mbar_wait(o_done, 0, abort_flag, status, kWaitCycles);
    tc_fence_after();
    float ow[16], ocm[16], os[16];
    tmem_ld16(lane_addr + kColOW, ow);
    tmem_ld16(lane_addr + kColOC, ocm);
    tmem_ld16(lane_addr + kColOS, os);
    tmem_ld_wait();
    if (r < D && !*abort_flag) {
      const int Hq = a.geo.Hq;
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        if (h >= G) break;
        const int gh = g * G + h;
        const float* gt = a.gates + ((size_t)b * Hq + gh) * 3;
        const float oc = it.ncc > 0 ? ocm[h] * inv_c[h] : 0.f;
        const float val = __ldg(gt + 0) * oc + __ldg(gt + 1) * os[h] * inv_s[h] +
                          __ldg(gt + 2) * ow[h] * inv_w[h];
        const size_t oi = ((size_t)b * Hq + gh) * D + r;
        if (a.geo.out_f32) {
          static_cast<float*>(a.out)[oi] = val;
        } else {
          const __nv_bfloat16 bv = __float2bfloat16_rn(val);
          static_cast<uint16_t*>(a.out)[oi] = *reinterpret_cast<const uint16_t*>(&bv);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_decode_t(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  using L = DecLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_decode_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  nsa_decode_kernel<D><<<a.batch * a.geo.Hkv, 192, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_compress(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)a.geo.l * a.geo.D * sizeof(float);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_decode_compress_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 128 * 4);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  nsa_decode_compress_kernel<<<dim3(a.batch, a.geo.Hkv, 2), 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s) {
  return a.geo.D == 128 ? launch_decode_t<128>(a, m, s) : launch_decode_t<64>(a, m, s);
}

}  // namespace nsa
