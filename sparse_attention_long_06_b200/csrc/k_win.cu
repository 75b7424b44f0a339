// Sliding-window attention (step 6) with its gate applied.
//
//   step 6 ("DeepSeek NSA config.toml" page, section 3, sliding_window; the
//   local-context branch of section 1): per query head, softmax over the w
//   tokens ending at t (t included) of s * q . k, output O_win = sum p v;
//   the kernel stores g_win * O_win (the gate of step 7, "DeepSeek NSA
//   config.toml" page, sections 1 and 3) as fp32 [T, Hq, D] for the selected
//   branch's epilogue to add.
//
// One persistent CTA per SM walks dense tiles of 128 MMA rows = (128 / G)
// consecutive tokens x the G query heads of one KV group (all tiles of group
// 0 first).  The tile's window keys [t0 - w + 1, t0 + 128 / G - 1] are shared
// by all of its rows and are streamed in chunks of 128 keys:
//   pass 1: S = Q K^T (rows on TMEM lanes), masked to each row's window:
//           row maximum;
//   pass 2: S again, P = exp(s - max) (largest element exactly 1, K-major A
//           operand in shared memory) and its row sum in fp32, O += P V in
//           TMEM; the epilogue scales row r by g_win / sum.
// Warp roles: 0 = TMA producer, 1 = tcgen05.mma issuer, 2..5 and 6..9 = two
// softmax warpgroups that take alternate key chunks of both passes (each with
// its own TMEM score buffer and P buffer) and split the epilogue's columns
// (thread i of warp w owns TMEM lane 32 * (w % 4) + i).
#include <type_traits>

#include "nsa_internal.cuh"
#include "sm100.cuh"

namespace nsa {
using namespace sm100;

namespace {

template <int D>
struct WinLayout {
  static constexpr int kStages = 3;
  static constexpr int kQBytes = kTileRows * D * 2;   // 128 rows
  static constexpr int kChunkBytes = kChunk * D * 2;  // 128 keys
  static constexpr int kPBytes = kTileRows * kChunk * 2;
  static constexpr int kQ = 0;                              // 2 buffers
  static constexpr int kRing = kQ + 2 * kQBytes;            // kStages
  static constexpr int kP = kRing + kStages * kChunkBytes;  // 2 buffers (one per warpgroup)
  static constexpr int kStat = kP + 2 * kPBytes;            // float m, l, m1, l1 [128]
  static constexpr int kBars = kStat + 4 * 128 * 4;
  static constexpr int kEnd = kBars + 32 * 8;
  // at least 116 KB so that one CTA owns an SM (it allocates all 512 TMEM columns)
  static constexpr int kSmem = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr int kWinThreads = 320;

struct WinItem {
  int valid, b, g, t0, T, row0, ntok, ws, nc, cu0, span;
};

// Keys of chunk c that lie in the tile's window span, rounded up to a
// multiple of 16 (the N of its QK^T and 16 x the K-steps of its PV): the
// last chunk of a span of w + 128/G - 1 keys is mostly empty.
__device__ __forceinline__ int chunk_width(const WinItem& it, int c) {
  const int rem = it.span - c * kChunk;
  return ((rem < kChunk ? rem : kChunk) + 15) & ~15;
}

__device__ __forceinline__ WinItem win_item(const PrefillArgs& a, int k) {
  WinItem it{};
  const int tiles = a.meta->tiles_total, H = a.geo.Hkv;
  if (k >= tiles * H) return it;
  it.valid = 1;
  it.g = k / tiles;  // group-major: one group's K/V stays hot in L2
  const int tau = k - it.g * tiles;
  it.b = seq_of_offset(a.tile_off, a.batch, tau);
  it.t0 = (tau - a.tile_off[it.b]) * a.geo.tpt;
  it.cu0 = __ldg(a.cu + it.b);
  it.T = __ldg(a.cu + it.b + 1) - it.cu0;
  it.row0 = it.cu0 + it.t0;
  it.ntok = min(a.geo.tpt, it.T - it.t0);
  it.ws = it.t0 - a.geo.w + 1;  // first window key of the tile's first token
  // keys [max(ws, 0), t0 + ntok - 1]; chunks start at ws (rounded down to 0 if
  // the whole window starts inside the sequence's first keys)
  const int first = max(it.ws, 0);
  it.ws = first == 0 ? 0 : it.ws;
  const int last = it.t0 + it.ntok - 1;
  it.span = last - it.ws + 1;
  it.nc = (it.span + kChunk - 1) / kChunk;
  return it;
}

template <int D>
__global__ void __launch_bounds__(kWinThreads, 1)
    nsa_win_kernel(const __grid_constant__ PrefillArgs a,
                   const __grid_constant__ PrefillMaps maps) {
  using L = WinLayout<D>;
  constexpr int KSTEPS = D / 16;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;     // [2]
  uint64_t* q_empty = bars + 2;    // [2]
  uint64_t* st_full = bars + 4;    // [3]
  uint64_t* st_empty = bars + 7;   // [3]
  uint64_t* s_full = bars + 10;    // [2] one TMEM score buffer per warpgroup
  uint64_t* s_empty = bars + 12;   // [2]
  uint64_t* p_full = bars + 14;    // [2] one P buffer per warpgroup
  uint64_t* p_empty = bars + 16;   // [2]
  uint64_t* o_full = bars + 18;
  uint64_t* o_empty = bars + 19;
  uint64_t* fin = bars + 20;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 22);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  float* m_s = reinterpret_cast<float*>(sm + L::kStat);  // merged row max (scaled, log2)
  float* l_s = m_s + 128;                                 // row sum, warpgroup 0's part
  float* m1_s = m_s + 256;
  float* l1_s = m_s + 384;                                // row sum, warpgroup 1's part

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (a.meta->bad) return;
  if (smem_u32(sm) & 1023u) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDeviceTimeoutCode);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, 4);
      mbar_init(p_full + i, 4);
      mbar_init(p_empty + i, 1);
    }
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, 8);
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
  const int G = a.geo.G;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k_win);
      tma_prefetch_desc(&maps.v_win);
      int qc = 0, sc = 0;
      bool ok = true;
      auto load_chunk = [&](const CUtensorMap* map, const WinItem& it, int c) {
        const int s = sc % L::kStages, u = sc / L::kStages;
        if (u > 0 && !mbar_wait(st_empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        uint8_t* dst = sm + L::kRing + s * L::kChunkBytes;
        mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(dst + h * 16384, map, st_full + s, h * 64, it.g, it.cu0 + it.ws + c * kChunk);
        ++sc;
      };
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const WinItem it = win_item(a, k);
        if (!it.valid) break;
        const int qb = qc & 1, u = qc >> 1;
        if (u > 0 && !mbar_wait(q_empty + qb, (u - 1) & 1, abort_flag, status, kWaitCycles)) break;
        mbar_arrive_expect_tx(q_full + qb, L::kQBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(sm + L::kQ + qb * L::kQBytes + h * 16384, &maps.q, q_full + qb, h * 64,
                      it.g * G, it.row0);
        ++qc;
        for (int c = 0; c < it.nc && ok; ++c) load_chunk(&maps.k_win, it, c);
        if (ok) load_chunk(&maps.k_win, it, 0);
        for (int c = 0; c < it.nc && ok; ++c) {
          if (c + 1 < it.nc) load_chunk(&maps.k_win, it, c + 1);
          if (ok) load_chunk(&maps.v_win, it, c);
        }
      }
      // drain: every issued copy has landed before the CTA retires (also
      // after an abort, hence a private never-set abort flag)
      volatile int never = 0;
      for (int s = 0; s < L::kStages && s < sc; ++s) {
        const int last = sc - 1 - ((sc - 1 - s) % L::kStages);
        mbar_wait(st_full + s, (last / L::kStages) & 1, &never, nullptr, kWaitCycles / 4);
      }
      for (int qb = 0; qb < 2 && qb < qc; ++qb) {
        const int last = qc - 1 - ((qc - 1 - qb) % 2);
        mbar_wait(q_full + qb, (last >> 1) & 1, &never, nullptr, kWaitCycles / 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_pv = idesc_bf16(128, D, false, true);
      int qc = 0, sc = 0, oc = 0;
      int s_use[2] = {0, 0}, p_use[2] = {0, 0};
      bool ok = true;
      // chunk c goes to TMEM score buffer c & 1 (owned by warpgroup c & 1)
      auto qk = [&](int qb, int c, int cw) {
        const uint32_t id_qk = idesc_bf16(128, cw, false, false);
        const int s = sc % L::kStages;
        if (!mbar_wait(st_full + s, (sc / L::kStages) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        const int buf = c & 1, u = s_use[buf];
        if (u > 0 && !mbar_wait(s_empty + buf, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t stage = sbase + L::kRing + s * L::kChunkBytes;
        const uint32_t qbuf = sbase + L::kQ + qb * L::kQBytes;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + buf * 128, smem_desc(qbuf + off, 16, 1024, kLayoutSw128),
                      smem_desc(stage + off, 16, 1024, kLayoutSw128), id_qk, ks > 0);
        }
        mma_commit(st_empty + s);
        mma_commit(s_full + buf);
        ++sc;
        ++s_use[buf];
      };
      auto pv = [&](int c, int cw) {
        const int s = sc % L::kStages, pb = c & 1;
        if (!mbar_wait(st_full + s, (sc / L::kStages) & 1, abort_flag, status, kWaitCycles) ||
            !mbar_wait(p_full + pb, p_use[pb] & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        if (c == 0 && oc > 0 && !mbar_wait(o_empty, (oc - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t stage = sbase + L::kRing + s * L::kChunkBytes;
        const uint32_t P = sbase + L::kP + pb * L::kPBytes;
        for (int ks = 0; ks < cw / 16; ++ks)
          mma_bf16_ss(tmem + 256, smem_desc(P + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSw128),
                      smem_desc(stage + ks * 2048, 16384, 1024, kLayoutSw128), id_pv,
                      (c > 0 || ks > 0) ? 1u : 0u);
        mma_commit(st_empty + s);
        mma_commit(p_empty + pb);
        ++sc;
        ++p_use[pb];
      };
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const WinItem it = win_item(a, k);
        if (!it.valid) break;
        const int qb = qc & 1;
        if (!mbar_wait(q_full + qb, (qc >> 1) & 1, abort_flag, status, kWaitCycles)) break;
        for (int c = 0; c < it.nc && ok; ++c) qk(qb, c, chunk_width(it, c));
        if (ok) qk(qb, 0, chunk_width(it, 0));
        for (int c = 0; c < it.nc && ok; ++c) {
          if (c + 1 < it.nc) qk(qb, c + 1, chunk_width(it, c + 1));
          if (ok) pv(c, chunk_width(it, c));
        }
        if (!ok) break;
        mma_commit(o_full);
        mma_commit(q_empty + qb);
        ++oc;
        ++qc;
      }
      mma_commit(fin);
      volatile int never = 0;
      mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Two warpgroups; warpgroup w handles the chunks c with c % 2 == w in both
    // passes and columns [w D/2, (w+1) D/2) of the output rows.
    const int w = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // TMEM lane = tile row owned by this thread
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const int Hq = a.geo.Hq, lgG = a.geo.lg_G, wlen = a.geo.w;
    int s_use = 0, p_use = 0, oc = 0;
    auto both_bar = [&]() { asm volatile("bar.sync 3, 256;" ::: "memory"); };
    for (int k = blockIdx.x;; k += gridDim.x) {
      const WinItem it = win_item(a, k);
      if (!it.valid) break;
      const int i_row = r >> lgG, h_row = r & (G - 1);
      const int t_row = it.t0 + i_row;
      const bool row_ok = i_row < it.ntok;
      // window keys of this row as offsets from the tile's first chunk key
      const int o_lo = max(t_row - wlen + 1, 0) - it.ws, o_hi = t_row - it.ws;
      const size_t orow = ((size_t)(it.row0 + i_row) * Hq + it.g * G + h_row);
      // ---- pass 1: row maximum over this warpgroup's chunks (scaled, log2 units)
      float m = -INFINITY;
      for (int c = w; c < it.nc; c += 2) {
        mbar_wait(s_full + w, s_use & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        const int lo = o_lo - c * kChunk, hi = o_hi - c * kChunk;
        // 16-column groups holding keys, and 64-column halves holding them
        // (tile-uniform: the TMEM loads below are warp-wide)
        const int ngc = chunk_width(it, c) >> 4;
        auto chunk_max = [&](auto full_tag) {
          constexpr bool kFull = decltype(full_tag)::value;
          const int ng = kFull ? 8 : ngc, nh = kFull ? 2 : (ngc + 3) >> 2;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (!kFull && half >= nh) break;
            float x[64];
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
              float v[16];
              if (kFull || half * 4 + g4 < ng) {
                tmem_ld16(lane_addr + w * 128 + half * 64 + g4 * 16, v);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;  // past the span: masked below
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) x[g4 * 16 + j] = v[j];
            }
            tmem_ld_wait();
            if (half == nh - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(s_empty + w);
            }
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const int o = half * 64 + j;
              if (row_ok && o >= lo && o <= hi) m = fmaxf(m, x[j]);
            }
          }
        };
        if (ngc == 8) chunk_max(std::true_type{});
        else chunk_max(std::false_type{});
        ++s_use;
      }
      m *= sl2;
      // merge the two warpgroups' row maxima
      if (w == 1) m1_s[r] = m;
      both_bar();  // every thread is also done with the previous tile's m_s / l_s / l1_s
      if (w == 0) m_s[r] = fmaxf(m, m1_s[r]);
      both_bar();
      const float mrow = m_s[r];
      float lsum = 0.f;  // this warpgroup's part of the row sum
      // ---- pass 2: P = exp2(s - max) into this warpgroup's P buffer (row r)
      for (int c = w; c < it.nc; c += 2) {
        mbar_wait(s_full + w, s_use & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        if (p_use > 0) mbar_wait(p_empty + w, (p_use - 1) & 1, abort_flag, status, kWaitCycles);
        const int lo = o_lo - c * kChunk, hi = o_hi - c * kChunk;
        const uint32_t prow = sbase + L::kP + w * L::kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
        const int ngc = chunk_width(it, c) >> 4;
        auto chunk_p = [&](auto full_tag) {
          constexpr bool kFull = decltype(full_tag)::value;
          const int ng = kFull ? 8 : ngc, nh = kFull ? 2 : (ngc + 3) >> 2;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (!kFull && half >= nh) break;
            float v[64];
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
              float u16[16];
              if (kFull || half * 4 + g4 < ng) {
                tmem_ld16(lane_addr + w * 128 + half * 64 + g4 * 16, u16);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) u16[j] = 0.f;
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) v[g4 * 16 + j] = u16[j];
            }
            tmem_ld_wait();
#pragma unroll
            for (int g8 = 0; g8 < 8; ++g8) {  // 8 keys per 16-byte chunk of the row
              if (!kFull && half * 8 + g8 >= 2 * ng) break;  // columns the PV does not read
              uint32_t pk[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int o0 = half * 64 + g8 * 8 + 2 * j;
                const float p0 = (row_ok && o0 >= lo && o0 <= hi) ? ex2(v[g8 * 8 + 2 * j] * sl2 - mrow) : 0.f;
                const float p1 = (row_ok && o0 + 1 >= lo && o0 + 1 <= hi)
                                     ? ex2(v[g8 * 8 + 2 * j + 1] * sl2 - mrow)
                                     : 0.f;
                lsum += p0 + p1;
                pk[j] = pack_bf16x2(p0, p1);
              }
              st_shared_v4(prow + half * 16384 + ((g8 ^ (r & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
            }
          }
        };
        if (ngc == 8) chunk_p(std::true_type{});
        else chunk_p(std::false_type{});
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(s_empty + w);
          mbar_arrive(p_full + w);
        }
        ++s_use;
        ++p_use;
      }
      // ---- epilogue: this warpgroup's half of the row, g_win * O / sum
      (w == 0 ? l_s : l1_s)[r] = lsum;
      both_bar();
      const float ls = l_s[r] + l1_s[r];
      mbar_wait(o_full, oc & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      const float gw = row_ok ? __ldg(a.gates + orow * 3 + 2) : 0.f;
      const float scale = ls > 0.f ? gw / ls : 0.f;
#pragma unroll
      for (int grp = 0; grp < D / 32; ++grp) {
        float v[16];
        tmem_ld16(lane_addr + 256 + w * (D / 2) + grp * 16, v);
        tmem_ld_wait();
        if (row_ok && !*abort_flag) {
          float4* o = reinterpret_cast<float4*>(a.o_win + orow * D + w * (D / 2) + grp * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o[j] = make_float4(v[4 * j] * scale, v[4 * j + 1] * scale, v[4 * j + 2] * scale,
                               v[4 * j + 3] * scale);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      ++oc;
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
cudaError_t launch_win_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                         cudaStream_t s) {
  using L = WinLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_win_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = num_sms < kMaxPersistentCtas ? num_sms : kMaxPersistentCtas;
  nsa_win_kernel<D><<<grid, kWinThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_win(const PrefillArgs& a, const PrefillMaps& m, int num_sms, cudaStream_t s) {
  return a.geo.D == 128 ? launch_win_t<128>(a, m, num_sms, s)
                        : launch_win_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
