// Compressed-branch attention and block scores (steps 2 and 3).
//
//   step 2 ("DeepSeek NSA config.toml" page, section 1: the compressed branch
//   gives coarse global context): per query head, softmax over the complete
//   compressed blocks of s * q . Kc, output O_cmp = sum p Vc;
//   step 3 ("DeepSeek NSA in manufacturing" page, section on what dynamic
//   sparsity sparsifies: the query's coarse attention to every compressed
//   block ranks the blocks): S[t, g, i] = sum over the heads of group g of p
//   for compressed block i (the top-n kernel sums these over each selection
//   block when the block sizes and stride differ).
// Compressed block i covers tokens [i d, i d + l - 1] and is visible to the
// queries t >= i d + l - 1.
//
// One persistent CTA per SM walks dense tiles of 128 MMA rows = (128 / G)
// consecutive tokens x the G query heads of one KV group.  The compressed
// keys are shared by all rows, so every product is a full 128 x 128 tcgen05
// tile.  Two passes over the compressed keys of the tile:
//   pass 1: S = Q Kc^T (rows = (token, head) on TMEM lanes): running max and
//           sum per row -> log-sum-exp;
//   pass 2: S^T = Kc Q^T (keys on TMEM lanes, (token, head) on columns):
//           p = exp(s - lse) is exact, the G columns of a token sum to its
//           block score inside one thread, P^T goes to shared memory as the
//           MN-major A operand of O = P Vc (accumulated in TMEM).
// Warp roles: 0 = TMA producer, 1 = tcgen05.mma issuer, 2..5 and 6..9 = two
// softmax warpgroups that take alternate key chunks of both passes (each
// with its own TMEM score buffer and P buffer) and split the epilogue's
// columns (thread i of warp w owns TMEM lane 32 * (w % 4) + i).
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"

namespace nsa {
using namespace sm100;

namespace {

template <int D>
struct CmpLayout {
  static constexpr int kStages = 3;
  static constexpr int kQBytes = kTileRows * D * 2;   // 128 rows
  static constexpr int kChunkBytes = kChunk * D * 2;  // 128 keys
  static constexpr int kPBytes = kChunk * kTileRows * 2;
  static constexpr int kQ = 0;                                   // 2 buffers
  static constexpr int kRing = kQ + 2 * kQBytes;                 // kStages
  static constexpr int kP = kRing + kStages * kChunkBytes;       // 2 buffers (one per warpgroup)
  static constexpr int kStat = kP + 2 * kPBytes;                 // float lse, sum, m1, l1 [128]
  static constexpr int kBars = kStat + 4 * 128 * 4;
  static constexpr int kEnd = kBars + 32 * 8;
  // at least 116 KB so that one CTA owns an SM (it allocates all 512 TMEM columns)
  static constexpr int kSmem = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr int kCmpThreads = 320;

struct CmpItem {
  int valid, b, g, t0, T, row0, nc, cmp0;
};

__device__ __forceinline__ CmpItem cmp_item(const PrefillArgs& a, int k) {
  CmpItem it{};
  const int tiles = a.meta->tiles_total, H = a.geo.Hkv;
  if (k >= tiles * H) return it;
  it.valid = 1;
  const int tau = tiles - 1 - k / H;  // heaviest (latest) tiles first
  it.g = k % H;
  it.b = seq_of_offset(a.tile_off, a.batch, tau);
  it.t0 = (tau - a.tile_off[it.b]) * a.geo.tpt;
  const int c0 = __ldg(a.cu + it.b);
  it.T = __ldg(a.cu + it.b + 1) - c0;
  it.row0 = c0 + it.t0;
  const int tend = min(it.t0 + a.geo.tpt, it.T);
  // compressed blocks visible to the tile's last token (t = tend - 1)
  const int ncmp_max = num_cmp_blocks(tend, a.geo.l, a.geo.d);
  it.nc = (ncmp_max + kChunk - 1) / kChunk;
  it.cmp0 = a.cmp_off[it.b];
  return it;
}

struct Pass2Rows {
  uint32_t taddr;        // TMEM address of this thread's score row (lane = key)
  const float* lse_s;    // per row: log2-sum-exp of the scaled scores
  const float* sum_s;    // per row: sum of exp2(s - row max)
  float sl2;             // softmax scale * log2(e)
  int row_lo, row_hi;    // rows (token * G + head) that see this key
  uint32_t prow;         // shared address of this key's row of P^T
  int r;                 // key within the chunk
  float* srow;           // block score of the tile's first token for this key
  size_t tok_stride;     // score elements between consecutive tokens
  volatile int* abort_flag;
};

// Pass 2 for one key and the 128 rows of a tile: p = exp2(s * sl2 - lse) per
// (token, head) row, the block score of each token = the sum of its G heads'
// p (the G heads of a token are G consecutive columns of this thread), and
// p * rowsum (= exp2(s - row max), largest element exactly 1) into P^T as
// bf16 in the 128-byte-swizzled MN-major layout.
template <int G, bool kFull>
__device__ __forceinline__ void pass2_rows(const Pass2Rows& a) {
  const bool live = !*a.abort_flag;
#pragma unroll
  for (int grp = 0; grp < kTileRows / 16; ++grp) {
    float v[16];
    tmem_ld16(a.taddr + grp * 16, v);
    tmem_ld_wait();
    float p[16], pm[16];
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 ls4 = *reinterpret_cast<const float4*>(a.lse_s + grp * 16 + j4 * 4);
      const float4 su4 = *reinterpret_cast<const float4*>(a.sum_s + grp * 16 + j4 * 4);
      const float lsv[4] = {ls4.x, ls4.y, ls4.z, ls4.w};
      const float suv[4] = {su4.x, su4.y, su4.z, su4.w};
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = j4 * 4 + jj;
        const int row = grp * 16 + j;
        p[j] = (kFull || (row >= a.row_lo && row < a.row_hi)) ? ex2(fmaf(v[j], a.sl2, -lsv[jj]))
                                                               : 0.f;
        pm[j] = p[j] * suv[jj];
      }
    }
#pragma unroll
    for (int kt = 0; kt < 16 / G; ++kt) {
      float ts = 0.f;
#pragma unroll
      for (int j = 0; j < G; ++j) ts += p[kt * G + j];
      const int row = grp * 16 + kt * G;
      if ((kFull || (row >= a.row_lo && row < a.row_hi)) && live)
        a.srow[(size_t)(row / G) * a.tok_stride] = ts;
    }
    uint32_t pk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(pm[2 * j], pm[2 * j + 1]);
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int cidx = grp * 2 + cc;
      const uint32_t addr = a.prow + (cidx >> 3) * 16384 + (((cidx & 7) ^ (a.r & 7)) << 4);
      st_shared_v4(addr, pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kCmpThreads, 1)
    nsa_cmp_attn_kernel(const __grid_constant__ PrefillArgs a,
                        const __grid_constant__ PrefillMaps maps) {
  using L = CmpLayout<D>;
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
  float* lse_s = reinterpret_cast<float*>(sm + L::kStat);
  float* sum_s = lse_s + 128;
  float* m1_s = lse_s + 256;
  float* l1_s = lse_s + 384;

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
  const int G = a.geo.G, l = a.geo.l, dstride = a.geo.d;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.kc);
      tma_prefetch_desc(&maps.vc);
      int qc = 0, sc = 0;
      bool ok = true;
      auto load_chunk = [&](const CUtensorMap* map, const CmpItem& it, int c) {
        const int s = sc % L::kStages, u = sc / L::kStages;
        if (u > 0 && !mbar_wait(st_empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles)) {
          ok = false;
          return;
        }
        uint8_t* dst = sm + L::kRing + s * L::kChunkBytes;
        mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(dst + h * 16384, map, st_full + s, h * 64, it.g, it.cmp0 + c * kChunk);
        ++sc;
      };
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const CmpItem it = cmp_item(a, k);
        if (!it.valid) break;
        if (it.nc == 0) continue;
        const int qb = qc & 1, u = qc >> 1;
        if (u > 0 && !mbar_wait(q_empty + qb, (u - 1) & 1, abort_flag, status, kWaitCycles)) break;
        mbar_arrive_expect_tx(q_full + qb, L::kQBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(sm + L::kQ + qb * L::kQBytes + h * 16384, &maps.q, q_full + qb, h * 64,
                      it.g * G, it.row0);
        ++qc;
        for (int c = 0; c < it.nc && ok; ++c) load_chunk(&maps.kc, it, c);
        if (ok) load_chunk(&maps.kc, it, 0);
        for (int c = 0; c < it.nc && ok; ++c) {
          if (c + 1 < it.nc) load_chunk(&maps.kc, it, c + 1);
          if (ok) load_chunk(&maps.vc, it, c);
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
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_bf16(128, D, true, true);
      int qc = 0, sc = 0, oc = 0;
      int s_use[2] = {0, 0}, p_use[2] = {0, 0};
      bool ok = true;
      // chunk c goes to TMEM score buffer c & 1 (owned by warpgroup c & 1);
      // pass 1: S = Q Kc^T, pass 2: S^T = Kc Q^T
      auto qk = [&](bool swapped, int qb, int c) {
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
        const uint32_t A = swapped ? stage : qbuf;
        const uint32_t B = swapped ? qbuf : stage;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + buf * 128, smem_desc(A + off, 16, 1024, kLayoutSw128),
                      smem_desc(B + off, 16, 1024, kLayoutSw128), id_qk, ks > 0);
        }
        mma_commit(st_empty + s);
        mma_commit(s_full + buf);
        ++sc;
        ++s_use[buf];
      };
      auto pv = [&](int c) {
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
#pragma unroll
        for (int ks = 0; ks < kChunk / 16; ++ks)
          mma_bf16_ss(tmem + 256, smem_desc(P + ks * 2048, 16384, 1024, kLayoutSw128),
                      smem_desc(stage + ks * 2048, 16384, 1024, kLayoutSw128), id_pv,
                      (c > 0 || ks > 0) ? 1u : 0u);
        mma_commit(st_empty + s);
        mma_commit(p_empty + pb);
        ++sc;
        ++p_use[pb];
      };
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const CmpItem it = cmp_item(a, k);
        if (!it.valid) break;
        if (it.nc == 0) continue;
        const int qb = qc & 1;
        if (!mbar_wait(q_full + qb, (qc >> 1) & 1, abort_flag, status, kWaitCycles)) break;
        for (int c = 0; c < it.nc && ok; ++c) qk(false, qb, c);
        if (ok) qk(true, qb, 0);
        for (int c = 0; c < it.nc && ok; ++c) {
          if (c + 1 < it.nc) qk(true, qb, c + 1);
          if (ok) pv(c);
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
    const int r = q4 * 32 + lane;  // TMEM lane owned by this thread
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const int Hq = a.geo.Hq, Hkv = a.geo.Hkv, cap = a.geo.cmp_cap, lgG = a.geo.lg_G;
    int s_use = 0, p_use = 0, oc = 0;
    auto group_bar = [&]() {
      if (w == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
      else asm volatile("bar.sync 2, 128;" ::: "memory");
    };
    auto both_bar = [&]() { asm volatile("bar.sync 3, 256;" ::: "memory"); };
    (void)group_bar;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const CmpItem it = cmp_item(a, k);
      if (!it.valid) break;
      const int i_row = r >> lgG, h_row = r & (G - 1);
      const int t_row = it.t0 + i_row;
      const bool row_ok = t_row < it.T;
      const int ncmp_row = row_ok ? num_cmp_blocks(t_row + 1, l, dstride) : 0;
      const size_t orow = ((size_t)(it.row0 + i_row) * Hq + it.g * G + h_row);
      if (it.nc == 0) {
        if (row_ok && !*abort_flag) {
          float4* o = reinterpret_cast<float4*>(a.o_cmp + orow * D + w * (D / 2));
          for (int j = 0; j < D / 8; ++j) o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (w == 0) a.lse[orow] = -INFINITY;
        }
        continue;
      }
      // ---- pass 1: running max / sum per row over this warpgroup's chunks
      float m = -INFINITY, lsum = 0.f;
      for (int c = w; c < it.nc; c += 2) {
        mbar_wait(s_full + w, s_use & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        const int jmax = ncmp_row - c * kChunk;  // columns j < jmax are visible blocks
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float x[64];
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            float v[16];
            tmem_ld16(lane_addr + w * 128 + half * 64 + g4 * 16, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) x[g4 * 16 + j] = v[j];
          }
          tmem_ld_wait();
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty + w);
          }
          float cm = -INFINITY;
          if (jmax >= (half + 1) * 64) {  // every column of this half is visible
#pragma unroll
            for (int j = 0; j < 64; ++j) cm = fmaxf(cm, x[j]);
            const float mn = fmaxf(m, cm * sl2);
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j) s += ex2(fmaf(x[j], sl2, -mn));
            lsum = lsum * ex2(m - mn) + s;
            m = mn;
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              x[j] = (half * 64 + j) < jmax ? x[j] * sl2 : -INFINITY;
              cm = fmaxf(cm, x[j]);
            }
            const float mn = fmaxf(m, cm);
            if (mn != -INFINITY) {
              float s = 0.f;
#pragma unroll
              for (int j = 0; j < 64; ++j) s += ex2(x[j] - mn);
              lsum = lsum * ex2(m - mn) + s;
              m = mn;
            }
          }
        }
        ++s_use;
      }
      // merge the two warpgroups' row statistics
      if (w == 1) {
        m1_s[r] = m;
        l1_s[r] = lsum;
      }
      both_bar();  // every thread is also done with the previous tile's lse_s / sum_s
      if (w == 0) {
        const float m1 = m1_s[r], l1 = l1_s[r];
        const float mm = fmaxf(m, m1);
        float ls = 0.f;
        if (mm != -INFINITY) ls = lsum * ex2(m - mm) + l1 * ex2(m1 - mm);
        lse_s[r] = ls > 0.f ? mm + __log2f(ls) : -INFINITY;
        sum_s[r] = ls;
      }
      both_bar();
      // ---- pass 2: this thread owns key r of this warpgroup's chunks
      for (int c = w; c < it.nc; c += 2) {
        mbar_wait(s_full + w, s_use & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        if (p_use > 0) mbar_wait(p_empty + w, (p_use - 1) & 1, abort_flag, status, kWaitCycles);
        const int key = c * kChunk + r;
        // rows (token, head) that see compressed block `key`: tokens t with
        // key * d + l - 1 <= t, inside the sequence
        const int tok_lo = max(0, key * dstride + l - 1 - it.t0);
        const int tok_hi = min(a.geo.tpt, it.T - it.t0);
        const int row_lo = tok_lo * G, row_hi = tok_hi * G;
        const uint32_t prow = sbase + L::kP + w * L::kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
        float* srow = a.scores + ((size_t)it.row0 * Hkv + it.g) * cap + key;
        const Pass2Rows rows{lane_addr + w * 128, lse_s, sum_s, sl2, row_lo, row_hi, prow, r,
                             srow, (size_t)Hkv * cap, abort_flag};
        // rows (token, head) of the tile all see every key of this warp: no
        // per-row test.  Warp-uniform, because pass2_rows issues warp-wide
        // (.sync.aligned) TMEM loads.
        const bool full = __all_sync(0xffffffffu, row_lo == 0 && row_hi == kTileRows);
        switch (lgG * 2 + (full ? 1 : 0)) {
          case 0: pass2_rows<1, false>(rows); break;
          case 1: pass2_rows<1, true>(rows); break;
          case 2: pass2_rows<2, false>(rows); break;
          case 3: pass2_rows<2, true>(rows); break;
          case 4: pass2_rows<4, false>(rows); break;
          case 5: pass2_rows<4, true>(rows); break;
          case 6: pass2_rows<8, false>(rows); break;
          case 7: pass2_rows<8, true>(rows); break;
          case 8: pass2_rows<16, false>(rows); break;
          default: pass2_rows<16, true>(rows); break;
        }
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
      // ---- epilogue: this warpgroup's half of the O_cmp row, and the LSE
      mbar_wait(o_full, oc & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      const float ls = sum_s[r];
      const float inv_sum = ls > 0.f ? 1.f / ls : 0.f;
#pragma unroll
      for (int grp = 0; grp < D / 32; ++grp) {
        float v[16];
        tmem_ld16(lane_addr + 256 + w * (D / 2) + grp * 16, v);
        tmem_ld_wait();
        if (row_ok && !*abort_flag) {
          float4* o = reinterpret_cast<float4*>(a.o_cmp + orow * D + w * (D / 2) + grp * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            o[j] = make_float4(v[4 * j] * inv_sum, v[4 * j + 1] * inv_sum, v[4 * j + 2] * inv_sum,
                               v[4 * j + 3] * inv_sum);
        }
      }
      if (w == 0 && row_ok && !*abort_flag) a.lse[orow] = lse_s[r] * 0.6931471805599453f;
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
cudaError_t launch_cmp_attn_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                              cudaStream_t s) {
  using L = CmpLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_cmp_attn_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = num_sms < kMaxPersistentCtas ? num_sms : kMaxPersistentCtas;
  nsa_cmp_attn_kernel<D><<<grid, kCmpThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cmp_attn(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                            cudaStream_t s) {
  return a.geo.D == 128 ? launch_cmp_attn_t<128>(a, m, num_sms, s)
                        : launch_cmp_attn_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
