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
// by all of its rows and are streamed once, in chunks of 128 keys (the last
// one only as wide as the keys it holds, rounded up to 16).  One pass with an
// online softmax:
//   S = Q K^T (rows on TMEM lanes), masked to each row's window; the chunk's
//   row maximum raises the running maximum m only when it grows by more than
//   2^8 (then the row's accumulator and sum are rescaled), so that most
//   chunks keep m; P = exp2(s - m) (bf16, K-major A operand in shared
//   memory), its row sum in fp32, O += P V in TMEM.
// Two softmax warpgroups take alternate key chunks, each with its own TMEM
// score buffer, P buffer, running (m, sum) and O accumulator; the epilogue
// merges the two accumulators of a row and stores g_win * O / sum.
// Warp roles (three warpgroups): 0 = TMA producer, 1 = tcgen05.mma issuer,
// 2..3 idle; 4..7 and 8..11 = the two softmax warpgroups (thread i of warp w
// owns TMEM lane 32 * (w % 4) + i; in the epilogue, softmax warpgroup w
// stores columns [w D/2, (w+1) D/2) of the rows).  The first warpgroup gives
// registers to the softmax warpgroups (setmaxnreg 56 / 224), which hold a
// whole 128-key row of scores in registers.
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
  static constexpr int kStat = kP + 2 * kPBytes;            // float m[2][128], l[2][128]
  static constexpr int kBars = kStat + 4 * 128 * 4;
  static constexpr int kEnd = kBars + 32 * 8;
  // at least 116 KB so that one CTA owns an SM (it allocates all 512 TMEM columns)
  static constexpr int kSmem = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr int kWinThreads = 384;
constexpr uint32_t kRegsControl = 56;   // producer / MMA warpgroup
constexpr uint32_t kRegsSoftmax = 224;  // softmax warpgroups: 56 + 2 * 224 = 3 * 168

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
  float* m_s = reinterpret_cast<float*>(sm + L::kStat);  // [warpgroup][row] running max (log2)
  float* l_s = m_s + 256;                                 // [warpgroup][row] running sum

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
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
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
        // the MMA issuer's order: K(0), then K(c) and V(c-1), then V(nc-1)
        load_chunk(&maps.k_win, it, 0);
        for (int c = 1; c < it.nc && ok; ++c) {
          load_chunk(&maps.k_win, it, c);
          if (ok) load_chunk(&maps.v_win, it, c - 1);
        }
        if (ok) load_chunk(&maps.v_win, it, it.nc - 1);
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
      // chunk c accumulates into the O of warpgroup c & 1 (TMEM columns
      // 256 + (c & 1) * D); the first chunk of each warpgroup overwrites it
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
        const uint32_t ocol = 256 + pb * D;
        for (int ks = 0; ks < cw / 16; ++ks)
          mma_bf16_ss(tmem + ocol, smem_desc(P + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSw128),
                      smem_desc(stage + ks * 2048, 16384, 1024, kLayoutSw128), id_pv,
                      (c > 1 || ks > 0) ? 1u : 0u);
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
        // QK^T of chunk c runs ahead of the PV of chunk c - 1
        qk(qb, 0, chunk_width(it, 0));
        for (int c = 1; c < it.nc && ok; ++c) {
          qk(qb, c, chunk_width(it, c));
          if (ok) pv(c - 1, chunk_width(it, c - 1));
        }
        if (ok) pv(it.nc - 1, chunk_width(it, it.nc - 1));
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
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax / epilogue
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // TMEM lane = tile row owned by this thread
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t o_col = 256 + w * D;  // this warpgroup's accumulator
    const float sl2 = a.geo.scale_log2;
    const int Hq = a.geo.Hq, lgG = a.geo.lg_G, wlen = a.geo.w;
    const int tpt = a.geo.tpt;
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
      // offsets seen by every row of the tile (tile-uniform)
      const int all_lo = max(it.t0 + tpt - 1 - wlen + 1, 0) - it.ws, all_hi = it.t0 - it.ws;
      const size_t orow = ((size_t)(it.row0 + i_row) * Hq + it.g * G + h_row);
      float m_run = -INFINITY;  // running maximum of s * scale * log2(e)
      float l_run = 0.f;        // sum of exp2(s * scale * log2(e) - m_run)
      for (int c = w; c < it.nc; c += 2) {
        mbar_wait(s_full + w, s_use & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        const int cw = chunk_width(it, c);
        const int ngc = cw >> 4;  // 16-column groups holding keys (tile-uniform)
        const bool full = it.ntok == tpt && cw == kChunk && all_lo <= c * kChunk &&
                          all_hi >= c * kChunk + kChunk - 1;
        float v[128];
#pragma unroll
        for (int g16 = 0; g16 < 8; ++g16) {
          float u16[16];
          if (g16 < ngc) {
            tmem_ld16(lane_addr + w * 128 + g16 * 16, u16);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) u16[j] = 0.f;  // past the chunk: masked below
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) v[g16 * 16 + j] = u16[j];
        }
        tmem_ld_wait();
        // the scores are in registers: the buffer can take the next chunk
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty + w);
        float cm = -INFINITY;
        if (full) {
#pragma unroll
          for (int j = 0; j < 128; ++j) cm = fmaxf(cm, v[j]);
        } else {
          const int lo = o_lo - c * kChunk, hi = o_hi - c * kChunk;
#pragma unroll
          for (int j = 0; j < 128; ++j) {
            v[j] = (row_ok && j >= lo && j <= hi) ? v[j] : -INFINITY;
            cm = fmaxf(cm, v[j]);
          }
        }
        cm *= sl2;
        // P buffer free, and the previous PV into this warpgroup's O done
        if (p_use > 0) mbar_wait(p_empty + w, (p_use - 1) & 1, abort_flag, status, kWaitCycles);
        // the maximum grew by more than 2^8: rescale the sum and O.  The TMEM
        // pass is warp-collective (.sync.aligned), so the whole warp takes it
        // when any of its rows needs it; the other rows scale by 1.
        const bool grow = cm > m_run + 8.f;
        const bool rescale = grow && m_run != -INFINITY;
        if (__any_sync(0xffffffffu, rescale)) {
          const float f = rescale ? ex2(m_run - cm) : 1.f;
          l_run *= f;
          tc_fence_after();
          // 16 columns at a time (the chunk's scores stay in registers)
          for (int g16 = 0; g16 < D / 16; ++g16) {
            float u16[16];
            tmem_ld16(lane_addr + o_col + g16 * 16, u16);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) u16[j] *= f;
            tmem_st16(lane_addr + o_col + g16 * 16, u16);
          }
          tmem_st_wait();
        }
        if (grow) m_run = cm;
        // P = exp2(s * sl2 - m_run): masked keys hold -inf and give 0 (and
        // when m_run is still -inf every key of the row is masked)
        const float nm = m_run == -INFINITY ? 0.f : -m_run;
        const uint32_t prow = sbase + L::kP + w * L::kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int g8 = 0; g8 < 16; ++g8) {  // 8 keys per 16-byte chunk of the row
          if (g8 >= 2 * ngc) break;        // columns the PV does not read
          uint32_t pk[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float p0 = ex2(fmaf(v[g8 * 8 + 2 * j], sl2, nm));
            const float p1 = ex2(fmaf(v[g8 * 8 + 2 * j + 1], sl2, nm));
            l_run += p0 + p1;
            pk[j] = pack_bf16x2(p0, p1);
          }
          st_shared_v4(prow + (g8 >> 3) * 16384 + (((g8 & 7) ^ (r & 7)) << 4), pk[0], pk[1], pk[2],
                       pk[3]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + w);
        ++s_use;
        ++p_use;
      }
      // ---- epilogue: merge the two warpgroups' (m, sum, O) of each row and
      // store this warpgroup's half of g_win * O / sum
      m_s[w * 128 + r] = m_run;
      l_s[w * 128 + r] = l_run;
      both_bar();
      const float m0 = m_s[r], m1 = m_s[128 + r], l0 = l_s[r], l1 = l_s[128 + r];
      both_bar();  // both have read: the arrays may be rewritten by the next tile
      const float mm = fmaxf(m0, m1);
      const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
      const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - mm);
      const float ls = l0 * f0 + l1 * f1;
      const bool has1 = it.nc > 1;  // warpgroup 1's accumulator was written this tile
      mbar_wait(o_full, oc & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      const float gw = row_ok ? __ldg(a.gates + orow * 3 + 2) : 0.f;
      const float scale = ls > 0.f ? gw / ls : 0.f;
      const float s0 = f0 * scale, s1 = f1 * scale;
#pragma unroll
      for (int grp = 0; grp < D / 32; ++grp) {
        const uint32_t col = w * (D / 2) + grp * 16;
        float x0[16], x1[16];
        tmem_ld16(lane_addr + 256 + col, x0);
        if (has1) {
          tmem_ld16(lane_addr + 256 + D + col, x1);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) x1[j] = 0.f;
        }
        tmem_ld_wait();
        if (row_ok && !*abort_flag) {
          float4* o = reinterpret_cast<float4*>(a.o_win + orow * D + col);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float e[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float y1 = has1 ? x1[4 * j + q] * s1 : 0.f;
              e[q] = x0[4 * j + q] * s0 + y1;
            }
            o[j] = make_float4(e[0], e[1], e[2], e[3]);
          }
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
  // the warpgroups' setmaxnreg shares add up to the launch allocation only
  // when the kernel is launched with 168 registers a thread: any other count
  // would leave setmaxnreg.inc waiting, so refuse to launch
  static int regs[64] = {};
  if (dev < 64 && regs[dev] == 0) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, nsa_win_kernel<D>);
    if (e != cudaSuccess) return e;
    regs[dev] = fa.numRegs;
  }
  if (dev < 64 && regs[dev] * (kWinThreads / 128) != kRegsControl + 2 * kRegsSoftmax)
    return cudaErrorInvalidConfiguration;
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
