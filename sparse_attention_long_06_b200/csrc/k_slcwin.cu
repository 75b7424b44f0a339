// Fused selected + sliding-window attention with the gate-combine epilogue
// (steps 5, 6 and 7).
//
//   step 5 ("DeepSeek NSA config.toml" page, section 3, select_block_size and
//   select_top_k; "DeepSeek NSA in manufacturing" page, section on what
//   dynamic sparsity sparsifies: token-level attention inside the selected
//   blocks): softmax over the tokens u <= t of the chosen blocks;
//   step 6 (config page, section 3, sliding_window): softmax over the w
//   tokens ending at t;
//   step 7 (config page, sections 1 and 3, learned gate aggregation):
//   out = g_cmp O_cmp + g_slc O_slc + g_win O_win.
//
// A persistent CTA per SM walks tiles of (128 / G) consecutive tokens of one
// KV group (all tiles of group 0 first, so that one group's K/V stays hot in
// L2).  Per tile:
//   window, as one dense 128-row tile shared by the tile's tokens:
//     pass A  S = Q K_win^T (rows on TMEM lanes): row max and sum;
//     pass B  S again, P = exp(S - max) into shared memory (K-major A
//             operand, largest element exactly 1), O_win += P V_win in TMEM;
//   selected, per token (its G heads share the index set): every selected
//     block is loaded once by TMA; S^T = K_blk Q_t^T (keys on TMEM lanes,
//     the token's heads on 16 columns), a two-sweep softmax over all of the
//     token's keys (block-wide max and sum per head), P^T into shared
//     memory, O_slc^T += V_blk^T P^T in TMEM.
// The MMA warp issues the QK^T of the next job before the PV of the current
// one, and the TMA warp loads in the same order, so that K/V streaming
// overlaps the softmax.  P is double-buffered.  A separate epilogue
// warpgroup turns O_win into g_win * O_win / sum rows of a per-CTA scratch
// slab (L2-resident) and writes each token's output
// g_cmp O_cmp + g_slc O_slc / sum + scratch, so that its global loads never
// sit on the softmax warps' path.
// Warp roles: 0 = TMA producer, 1 = tcgen05.mma issuer, 2..5 = softmax,
// 6..9 = epilogue (warp w owns TMEM lanes 32 * (w % 4) .. + 31).
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "softmax_util.cuh"

namespace nsa {
using namespace sm100;

namespace {

template <int D>
struct SwLayout {
  static constexpr int kStages = 4;
  static constexpr int kQBytes = kTileRows * D * 2;
  static constexpr int kChunkBytes = kChunk * D * 2;
  static constexpr int kPBytes = kChunk * kTileRows * 2;
  // B-operand row windows of the selected branch may run 8 rows past the Q
  // tile; they land in ring stage 0 (in bounds, and only in ignored columns)
  static constexpr int kQ = 0;
  static constexpr int kRing = kQBytes;
  static constexpr int kP = kRing + kStages * kChunkBytes;  // 2 buffers
  static constexpr int kRed = kP + 2 * kPBytes;            // float[2][16][4]
  static constexpr int kWstat = kRed + 2 * 16 * 4 * 4;     // float[128]
  static constexpr int kInv = kWstat + 128 * 4;            // float[2][16]
  static constexpr int kBars = kInv + 2 * 16 * 4;          // barriers + flags
  static constexpr int kEnd = kBars + 34 * 8;
  static constexpr int kSmem = kEnd + 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr uint32_t kColOwin = 256;
constexpr uint32_t kColOslc = 384;
constexpr int kThreads = 320;

struct SwTile {
  int valid, k, b, g, t0, T, row0, ntok, nwc, ws, nsc, njobs;
};

__device__ __forceinline__ SwTile sw_tile(const PrefillArgs& a, int k) {
  SwTile t{};
  const int tiles = a.meta->tiles_total, H = a.geo.Hkv;
  if (k >= tiles * H) return t;
  t.valid = 1;
  t.k = k;
  t.g = k / tiles;  // group-major
  const int tau = k - t.g * tiles;
  t.b = seq_of_offset(a.tile_off, a.batch, tau);
  t.t0 = (tau - a.tile_off[t.b]) * a.geo.tpt;
  const int c0 = __ldg(a.cu + t.b);
  t.T = __ldg(a.cu + t.b + 1) - c0;
  t.row0 = c0 + t.t0;
  t.ntok = min(a.geo.tpt, t.T - t.t0);
  t.nwc = (a.geo.w + a.geo.tpt - 1 + kChunk - 1) / kChunk;
  t.ws = t.t0 - a.geo.w + 1;
  const int bpc = kChunk >> a.geo.lg_l;
  t.nsc = (a.geo.n + bpc - 1) / bpc;
  t.njobs = 2 * t.nwc + t.ntok;
  return t;
}

// job types inside a tile: [0, nwc) window pass A, [nwc, 2 nwc) window pass B,
// [2 nwc, njobs) one selected-branch job per token
enum { kJobWinA = 0, kJobWinB = 1, kJobTok = 2 };
__device__ __forceinline__ int job_type(const SwTile& t, int jb) {
  return jb < t.nwc ? kJobWinA : (jb < 2 * t.nwc ? kJobWinB : kJobTok);
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__device__ __forceinline__ void reduce16(float (&v)[16], float* red, int q4, int lane,
                                         bool is_max) {
  reduce16_across_128<1>(v, red, q4, lane, is_max);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    nsa_slc_win_kernel(const __grid_constant__ PrefillArgs a,
                       const __grid_constant__ PrefillMaps maps) {
  using L = SwLayout<D>;
  constexpr int KSTEPS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* st_full = bars + 2;      // [4]
  uint64_t* st_empty = bars + 6;     // [4]
  uint64_t* s_full = bars + 10;      // [2]
  uint64_t* s_empty = bars + 12;     // [2]
  uint64_t* p_full = bars + 14;      // [2]
  uint64_t* p_empty = bars + 16;     // [2]
  uint64_t* owin_full = bars + 18;
  uint64_t* owin_empty = bars + 19;  // epilogue done with O_win and the window stats
  uint64_t* wstat_full = bars + 20;
  uint64_t* oslc_full = bars + 21;   // [2]
  uint64_t* tok_ready = bars + 23;   // [2] softmax wrote the token's 1/sum
  uint64_t* tok_done = bars + 25;    // [2] epilogue done with O_slc[slot] and 1/sum
  uint64_t* fin = bars + 27;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 30);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 31);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  float* wstat = reinterpret_cast<float*>(sm + L::kWstat);
  float* inv_s = reinterpret_cast<float*>(sm + L::kInv);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (a.meta->bad) return;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, 4);
      mbar_init(p_full + i, 4);
      mbar_init(p_empty + i, 1);
      mbar_init(oslc_full + i, 1);
      mbar_init(tok_ready + i, 4);
      mbar_init(tok_done + i, 4);
    }
    mbar_init(owin_full, 1);
    mbar_init(owin_empty, 4);
    mbar_init(wstat_full, 4);
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
  const int G = a.geo.G, l = a.geo.l, n = a.geo.n, Hkv = a.geo.Hkv, Hq = a.geo.Hq;
  const int lg_l = a.geo.lg_l;
  const int bpc = kChunk >> lg_l;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k_win);
      tma_prefetch_desc(&maps.v_win);
      tma_prefetch_desc(&maps.k_blk);
      tma_prefetch_desc(&maps.v_blk);
      int qc = 0, sc = 0;
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
      auto load_win = [&](const SwTile& t, int c, bool is_v) {
        uint8_t* dst = acquire();
        if (!dst) return;
        const int s = sc % L::kStages;
        const int row = __ldg(a.cu + t.b) + t.ws + c * kChunk;
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(dst + h * 16384, is_v ? &maps.v_win : &maps.k_win, st_full + s, h * 64, t.g, row);
        ++sc;
      };
      auto load_sel = [&](const SwTile& t, int i, bool is_v) {
        const int* sel = a.sel + ((size_t)(t.row0 + i) * Hkv + t.g) * n;
        const int c0 = __ldg(a.cu + t.b);
        for (int c = 0; c < t.nsc && ok; ++c) {
          uint8_t* dst = acquire();
          if (!dst) return;
          const int s = sc % L::kStages;
          for (int sub = 0; sub < bpc; ++sub) {
            const int bs = c * bpc + sub;
            const int blk = bs < n ? sel[bs] : -1;
            const int row = blk >= 0 ? c0 + (blk << lg_l) : -(1 << 24);
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(dst + h * 16384 + sub * l * 128, is_v ? &maps.v_blk : &maps.k_blk,
                          st_full + s, h * 64, t.g, row);
          }
          ++sc;
        }
      };
      auto load_q = [&](const SwTile& t) {
        if (qc > 0 && !mbar_wait(q_empty, (qc - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(sm + L::kQ + h * 16384, &maps.q, q_full, h * 64, t.g * G, t.row0);
        ++qc;
      };
      auto load_k = [&](const SwTile& t, int jb) {
        const int ty = job_type(t, jb);
        if (ty == kJobWinA) load_win(t, jb, false);
        else if (ty == kJobWinB) load_win(t, jb - t.nwc, false);
        else load_sel(t, jb - 2 * t.nwc, false);
      };
      auto load_v = [&](const SwTile& t, int jb) {
        const int ty = job_type(t, jb);
        if (ty == kJobWinB) load_win(t, jb - t.nwc, true);
        else if (ty == kJobTok) load_sel(t, jb - 2 * t.nwc, true);
      };
      SwTile cur = sw_tile(a, blockIdx.x);
      int jb = 0;
      if (cur.valid) {
        load_q(cur);
        if (ok) load_k(cur, 0);
        while (ok) {
          SwTile nt = cur;
          int njb = jb + 1;
          if (njb >= cur.njobs) {
            nt = sw_tile(a, cur.k + gridDim.x);
            njb = 0;
          }
          if (nt.valid) {
            if (njb == 0) load_q(nt);
            if (ok) load_k(nt, njb);
          }
          if (ok) load_v(cur, jb);
          if (!nt.valid) break;
          cur = nt;
          jb = njb;
        }
      }
      volatile int never = 0;
      for (int s = 0; s < L::kStages && s < sc; ++s) {
        const int last = sc - 1 - ((sc - 1 - s) % L::kStages);
        mbar_wait(st_full + s, (last / L::kStages) & 1, &never, nullptr, kWaitCycles / 4);
      }
      if (qc > 0) mbar_wait(q_full, (qc - 1) & 1, &never, nullptr, kWaitCycles / 4);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_win_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_win_pv = idesc_bf16(128, D, false, true);
      constexpr uint32_t id_slc_qk = idesc_bf16(128, 16, false, false);
      constexpr uint32_t id_slc_pv = idesc_bf16(128, 16, true, true);
      const uint32_t Qs = sbase + L::kQ, Ps = sbase + L::kP;
      int qc = 0, sc = 0, sbc = 0, pc = 0, owc = 0, tc = 0;
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
      auto release_stage = [&]() {
        mma_commit(st_empty + (sc % L::kStages));
        ++sc;
      };
      auto qk = [&](const SwTile& t, int jb) {
        const int ty = job_type(t, jb);
        const int buf = sbc & 1, u = sbc >> 1;
        if (u > 0 && !mbar_wait(s_empty + buf, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        const uint32_t dcol = tmem + buf * 128;
        if (ty != kJobTok) {
          const uint32_t st = wait_stage();
          if (!ok) return;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_bf16_ss(dcol, smem_desc(Qs + off, 16, 1024, kLayoutSw128),
                        smem_desc(st + off, 16, 1024, kLayoutSw128), id_win_qk, ks > 0);
          }
          release_stage();
        } else {
          const int i = jb - 2 * t.nwc;
          const uint32_t qrow = Qs + ((i * G) >> 3) * 1024;
          for (int c = 0; c < t.nsc && ok; ++c) {
            const uint32_t st = wait_stage();
            if (!ok) return;
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
              const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
              mma_bf16_ss(dcol + c * 16, smem_desc(st + off, 16, 1024, kLayoutSw128),
                          smem_desc(qrow + off, 16, 1024, kLayoutSw128), id_slc_qk, ks > 0);
            }
            release_stage();
          }
        }
        mma_commit(s_full + buf);
        ++sbc;
      };
      auto pv = [&](const SwTile& t, int jb) {
        const int ty = job_type(t, jb);
        if (ty == kJobWinA) return;
        const int pb = pc & 1;
        if (!mbar_wait(p_full + pb, (pc >> 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        const uint32_t P = Ps + pb * L::kPBytes;
        if (ty == kJobWinB) {
          const int c = jb - t.nwc;
          if (c == 0 && owc > 0 &&
              !mbar_wait(owin_empty, (owc - 1) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            return;
          }
          const uint32_t st = wait_stage();
          if (!ok) return;
#pragma unroll
          for (int ks = 0; ks < kChunk / 16; ++ks) {
            const uint32_t aoff = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_bf16_ss(tmem + kColOwin, smem_desc(P + aoff, 16, 1024, kLayoutSw128),
                        smem_desc(st + ks * 2048, 16384, 1024, kLayoutSw128), id_win_pv,
                        (c > 0 || ks > 0) ? 1u : 0u);
          }
          release_stage();
          mma_commit(p_empty + pb);
          ++pc;
          if (c == t.nwc - 1) {
            mma_commit(owin_full);
            ++owc;
          }
        } else {
          const int slot = tc & 1, u = tc >> 1;
          if (u > 0 && !mbar_wait(tok_done + slot, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            return;
          }
          for (int c = 0; c < t.nsc && ok; ++c) {
            const uint32_t st = wait_stage();
            if (!ok) return;
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks)
              mma_bf16_ss(tmem + kColOslc + slot * 16,
                          smem_desc(st + ks * 2048, 16384, 1024, kLayoutSw128),
                          smem_desc(P + c * 4096 + ks * 256, 128, 2048, kLayoutNone), id_slc_pv,
                          (c > 0 || ks > 0) ? 1u : 0u);
            release_stage();
          }
          mma_commit(p_empty + pb);
          ++pc;
          mma_commit(oslc_full + slot);
          ++tc;
        }
      };
      SwTile cur = sw_tile(a, blockIdx.x);
      int jb = 0;
      if (cur.valid) {
        if (!mbar_wait(q_full, qc & 1, abort_flag, status, kWaitCycles)) ok = false;
        tc_fence_after();
        if (ok) qk(cur, 0);
        while (ok) {
          SwTile nt = cur;
          int njb = jb + 1;
          if (njb >= cur.njobs) {
            nt = sw_tile(a, cur.k + gridDim.x);
            njb = 0;
          }
          if (nt.valid) {
            if (njb == 0) {
              // every QK of the current tile is issued: its Q buffer may be refilled
              mma_commit(q_empty);
              ++qc;
              if (!mbar_wait(q_full, qc & 1, abort_flag, status, kWaitCycles)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            qk(nt, njb);
          }
          if (ok) pv(cur, jb);
          if (!nt.valid) break;
          cur = nt;
          jb = njb;
        }
      }
      mma_commit(fin);
      volatile int never = 0;
      mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const int w = a.geo.w;
    int sbc = 0, pc = 0, tcs = 0, tiles_done = 0;
    auto wait_s = [&]() -> int {
      const int buf = sbc & 1;
      mbar_wait(s_full + buf, (sbc >> 1) & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      return buf;
    };
    auto release_s = [&](int buf, bool with_p, int pb) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(s_empty + buf);
        if (with_p) mbar_arrive(p_full + pb);
      }
      ++sbc;
    };
    // claims the next P buffer: waits until the MMA finished reading its last use
    auto claim_p = [&]() -> int {
      const int pb = pc & 1, u = pc >> 1;
      if (u > 0) mbar_wait(p_empty + pb, (u - 1) & 1, abort_flag, status, kWaitCycles);
      ++pc;
      return pb;
    };
    const int key_in_blk = r & (l - 1), slot_in_chunk = r >> lg_l;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const SwTile t = sw_tile(a, k);
      if (!t.valid) break;
      const int i_row = r >> a.geo.lg_G;
      const bool row_ok = i_row < t.ntok;
      // window keys of this row, as offsets into the tile's window span
      const int o_lo = max(i_row, -t.ws), o_hi = i_row + w - 1;
      // ---- window pass A: row max and sum
      float m = -INFINITY, lsum = 0.f;
      for (int c = 0; c < t.nwc; ++c) {
        const int buf = wait_s();
        float x[kChunk];
#pragma unroll
        for (int grp = 0; grp < kChunk / 16; ++grp) {
          float v[16];
          tmem_ld16(lane_addr + buf * 128 + grp * 16, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) x[grp * 16 + j] = v[j];
        }
        tmem_ld_wait();
        release_s(buf, false, 0);
        const int lo = o_lo - c * kChunk, hi = o_hi - c * kChunk;
        float cm = -INFINITY;
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          x[j] = (row_ok && j >= lo && j <= hi) ? x[j] * sl2 : -INFINITY;
          cm = fmaxf(cm, x[j]);
        }
        const float mn = fmaxf(m, cm);
        if (mn != -INFINITY) {
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < kChunk; ++j) s += ex2(x[j] - mn);
          lsum = lsum * ex2(m - mn) + s;
          m = mn;
        }
      }
      // 1 / row sum for the window epilogue (after it released the previous tile's)
      if (tiles_done > 0) mbar_wait(owin_empty, (tiles_done - 1) & 1, abort_flag, status, kWaitCycles);
      wstat[r] = lsum > 0.f ? 1.f / lsum : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(wstat_full);
      // ---- window pass B: P = exp(s - max), O_win += P V (in the MMA warp)
      for (int c = 0; c < t.nwc; ++c) {
        const int buf = wait_s();
        const int pb = claim_p();
        const int lo = o_lo - c * kChunk, hi = o_hi - c * kChunk;
        const uint32_t prow = sbase + L::kP + pb * L::kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float v[64];
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            float u16[16];
            tmem_ld16(lane_addr + buf * 128 + half * 64 + g4 * 16, u16);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[g4 * 16 + j] = u16[j];
          }
          tmem_ld_wait();
#pragma unroll
          for (int g8 = 0; g8 < 8; ++g8) {  // 8 keys per 16-byte chunk
            uint32_t pk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int j0 = half * 64 + g8 * 8 + 2 * j;
              const float p0 = (row_ok && j0 >= lo && j0 <= hi) ? ex2(v[g8 * 8 + 2 * j] * sl2 - m) : 0.f;
              const float p1 = (row_ok && j0 + 1 >= lo && j0 + 1 <= hi) ? ex2(v[g8 * 8 + 2 * j + 1] * sl2 - m) : 0.f;
              pk[j] = pack_bf16x2(p0, p1);
            }
            const uint32_t addr = prow + half * 16384 + ((g8 ^ (r & 7)) << 4);
            st_shared_v4(addr, pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_async_smem();
        release_s(buf, true, pb);
      }
      ++tiles_done;
      // ---- selected branch, one job per token; this thread owns key lane r
      const int* selbase = a.sel + ((size_t)t.row0 * Hkv + t.g) * n;
      // block index of this thread's key in every chunk, loaded one token ahead
      int blk_next[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int bs = c * bpc + slot_in_chunk;
        blk_next[c] = (t.ntok > 0 && c < t.nsc && bs < n) ? __ldg(selbase + bs) : -1;
      }
      for (int i = 0; i < t.ntok; ++i) {
        const int tt = t.t0 + i;
        bool kok[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) kok[c] = blk_next[c] >= 0 && (blk_next[c] << lg_l) + key_in_blk <= tt;
        if (i + 1 < t.ntok) {
          const int* seln = selbase + (size_t)(i + 1) * Hkv * n;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int bs = c * bpc + slot_in_chunk;
            blk_next[c] = (c < t.nsc && bs < n) ? __ldg(seln + bs) : -1;
          }
        }
        const int buf = wait_s();
        float mx[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
        // sweep 1: per-column maximum over this thread's keys
#pragma unroll
        for (int c0 = 0; c0 < 8; c0 += 4) {
          if (c0 >= t.nsc) break;
          float v[64];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float u16[16];
            tmem_ld16(lane_addr + buf * 128 + (c0 + cc) * 16, u16);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[cc * 16 + j] = u16[j];
          }
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            if (c0 + cc < t.nsc && kok[c0 + cc]) {
#pragma unroll
              for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[cc * 16 + h] * sl2);
            }
          }
        }
        reduce16(mx, red, q4, lane, true);
        // sweep 2: probabilities, column sums, P^T chunks
        const int pb = claim_p();
        const uint32_t pbase = sbase + L::kP + pb * L::kPBytes + (r >> 3) * 128 + (r & 7) * 16;
        float sm16[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) sm16[h] = 0.f;
        const int co = (i * G) & 7;
        uint32_t colmask = 0;  // columns that hold this token's heads
#pragma unroll
        for (int h = 0; h < 16; ++h) colmask |= (h >= co && h < co + G) ? (1u << h) : 0u;
#pragma unroll
        for (int c0 = 0; c0 < 8; c0 += 4) {
          if (c0 >= t.nsc) break;
          float v[64];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float u16[16];
            tmem_ld16(lane_addr + buf * 128 + (c0 + cc) * 16, u16);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[cc * 16 + j] = u16[j];
          }
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c = c0 + cc;
            if (c >= t.nsc) break;
            float p[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
              p[h] = (kok[c] && ((colmask >> h) & 1u)) ? ex2(v[cc * 16 + h] * sl2 - mx[h]) : 0.f;
              sm16[h] += p[h];
            }
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
            st_shared_v4(pbase + c * 4096, pk[0], pk[1], pk[2], pk[3]);
            st_shared_v4(pbase + c * 4096 + 2048, pk[4], pk[5], pk[6], pk[7]);
          }
        }
        fence_async_smem();
        release_s(buf, true, pb);
        reduce16(sm16, red + 64, q4, lane, false);
        // 1 / column sum for the epilogue warps (after they released this slot)
        const int slot = tcs & 1, u = tcs >> 1;
        if (u > 0) mbar_wait(tok_done + slot, (u - 1) & 1, abort_flag, status, kWaitCycles);
        if (r < 16) {
          float sv = 0.f;
#pragma unroll
          for (int h = 0; h < 16; ++h) sv = (h == r) ? sm16[h] : sv;
          inv_s[slot * 16 + r] = (((colmask >> r) & 1u) && sv > 0.f) ? 1.f / sv : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(tok_ready + slot);
        ++tcs;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float* scratch = a.scratch + (size_t)blockIdx.x * a.geo.tpt * G * D;
    int tiles_done = 0, tce = 0;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const SwTile t = sw_tile(a, k);
      if (!t.valid) break;
      // ---- window: g_win * O_win / sum rows into the scratch slab (lane = row)
      const int i_row = r >> a.geo.lg_G, h_row = r & (G - 1);
      const bool row_ok = i_row < t.ntok;
      const size_t tg_row = (size_t)t.row0 + i_row;
      const float gw = row_ok ? __ldg(a.gates + (tg_row * Hq + t.g * G + h_row) * 3 + 2) : 0.f;
      epilogue_bar();  // the previous tile's token outputs are done with the slab
      mbar_wait(wstat_full, tiles_done & 1, abort_flag, status, kWaitCycles);
      mbar_wait(owin_full, tiles_done & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      const float scale = gw * wstat[r];
#pragma unroll
      for (int g4 = 0; g4 < D / 64; ++g4) {
        float v[64];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float u16[16];
          tmem_ld16(lane_addr + kColOwin + g4 * 64 + cc * 16, u16);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[cc * 16 + j] = u16[j];
        }
        tmem_ld_wait();
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(scratch + (size_t)r * D + g4 * 64);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            dst[j] = make_float4(scale * v[4 * j], scale * v[4 * j + 1], scale * v[4 * j + 2],
                                 scale * v[4 * j + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(owin_empty);
      ++tiles_done;
      __threadfence_block();
      epilogue_bar();  // slab rows visible to every epilogue thread
      // ---- tokens: lane = channel
      for (int i = 0; i < t.ntok; ++i) {
        const int slot = tce & 1, ph = (tce >> 1) & 1;
        mbar_wait(tok_ready + slot, ph, abort_flag, status, kWaitCycles);
        mbar_wait(oslc_full + slot, ph, abort_flag, status, kWaitCycles);
        tc_fence_after();
        float o[16];
        tmem_ld16(lane_addr + kColOslc + slot * 16, o);
        tmem_ld_wait();
        float inv[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) inv[h] = inv_s[slot * 16 + h];
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tok_done + slot);
        ++tce;
        if (r < D && !*abort_flag) {
          const int co = (i * G) & 7;
          const size_t tg = (size_t)t.row0 + i;
#pragma unroll
          for (int col = 0; col < 16; ++col) {
            const int h = col - co;
            if (h < 0 || h >= G) continue;
            const int gh = t.g * G + h;
            const float* gt = a.gates + (tg * Hq + gh) * 3;
            const float val = __ldg(gt + 0) * a.o_cmp[(tg * Hq + gh) * D + r] +
                              __ldg(gt + 1) * o[col] * inv[col] +
                              scratch[(i * G + h) * D + r];
            const size_t oi = (tg * Hq + gh) * D + r;
            if (a.geo.out_f32) {
              static_cast<float*>(a.out)[oi] = val;
            } else {
              const __nv_bfloat16 bv = __float2bfloat16_rn(val);
              static_cast<uint16_t*>(a.out)[oi] = *reinterpret_cast<const uint16_t*>(&bv);
            }
          }
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
cudaError_t launch_slc_win_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                             cudaStream_t s) {
  using L = SwLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_slc_win_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = num_sms < kMaxPersistentCtas ? num_sms : kMaxPersistentCtas;
  nsa_slc_win_kernel<D><<<grid, kThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_slc_win(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                           cudaStream_t s) {
  return a.geo.D == 128 ? launch_slc_win_t<128>(a, m, num_sms, s)
                        : launch_slc_win_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
