// Select-only block attention (MoBA style): block mean keys and routing
// scores.
//
// "NSA vs MoBA" page (gtnt.cn/news/122266), section 1: MoBA cuts the
// sequence into blocks and a gate routes every query to a few key blocks,
// the way a mixture of experts routes tokens.  Here a block's routing key is
// the mean of its l' keys (bf16), and the routing score of block j for token
// t and KV group g is the sum over the group's query heads of q . mean key.
// The query's own block is always attended and n - 1 more are chosen by
// score (top-n kernel); the attention itself is the selected-block kernel
// without the other branches.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"

namespace nsa {
using namespace sm100;

// ------------------------------------------------------------------ mean keys
// Kbar[r, h, c] = bf16(sum_{p < l'} K[tok0(r) + p, h, c] / l') for every
// complete block r of every sequence.  The sum runs in fp64 in token order,
// so it is exact for any bf16 inputs whose exponents span less than about 40
// binades, and the division by a power of two is exact: the stored key is
// the mean rounded once to nearest even.  One thread per (block, head, 8
// channels), 16-byte loads.  Rows in [blocks, rows) are zero-filled.
__global__ void __launch_bounds__(256) nsa_block_mean_kernel(PrefillArgs a) {
  if (a.meta->bad) return;
  const int H = a.geo.Hkv, D = a.geo.D, L = a.geo.ls;
  const int per_row = H * (D / 8);
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.cmp_rows * per_row) return;
  const int r = (int)(idx / per_row);
  const int rem = (int)(idx % per_row);
  const int h = rem / (D / 8), c0 = (rem % (D / 8)) * 8;
  uint16_t* dst = a.k_cmp + ((size_t)r * H + h) * D + c0;
  if (r >= a.meta->cmp_total) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int b = seq_of_offset(a.cmp_off, a.batch, r);
  const int tok0 = __ldg(a.cu + b) + (r - a.cmp_off[b]) * L;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  const uint16_t* src = a.k + ((size_t)tok0 * H + h) * D + c0;
  for (int p = 0; p < L; ++p) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + (size_t)p * H * D));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += (double)__uint_as_float(w[e] << 16);
      acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
  const double inv = 1.0 / (double)L;  // a power of two: exact
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 lo = __double2bfloat16(acc[2 * e] * inv);
    const __nv_bfloat16 hi = __double2bfloat16(acc[2 * e + 1] * inv);
    o[e] = (uint32_t)*reinterpret_cast<const uint16_t*>(&lo) |
           ((uint32_t)*reinterpret_cast<const uint16_t*>(&hi) << 16);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_block_mean(const PrefillArgs& a, cudaStream_t s) {
  const long long threads = (long long)a.cmp_rows * a.geo.Hkv * (a.geo.D / 8);
  if (threads <= 0) return cudaSuccess;
  nsa_block_mean_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

// Decode: when the newest token completes its block (len % l' == 0), that
// block's mean key (fp64 sum in token order, rounded once) goes into the
// mean-key cache [B, cap / l', Hkv, D] for the steps that follow.  One CTA
// per (sequence, KV head), one thread per 8 channels.
__global__ void nsa_decode_block_mean_kernel(DecodeArgs a) {
  const int b = blockIdx.x, h = blockIdx.y, D = a.geo.D, H = a.geo.Hkv, L = a.geo.ls;
  const int c0 = threadIdx.x * 8;
  if (c0 >= D) return;
  const int len = __ldg(a.seqlens + b);
  if (len < L || len > a.cap || len % L != 0) return;
  const int j = len / L - 1;
  const uint16_t* src = a.k_cache + (((size_t)b * a.cap + (size_t)j * L) * H + h) * D + c0;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  for (int p = 0; p < L; ++p) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + (size_t)p * H * D));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += (double)__uint_as_float(w[e] << 16);
      acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
  const double inv = 1.0 / (double)L;
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 lo = __double2bfloat16(acc[2 * e] * inv);
    const __nv_bfloat16 hi = __double2bfloat16(acc[2 * e + 1] * inv);
    o[e] = (uint32_t)*reinterpret_cast<const uint16_t*>(&lo) |
           ((uint32_t)*reinterpret_cast<const uint16_t*>(&hi) << 16);
  }
  uint16_t* dst = a.k_cmp + (((size_t)b * a.ccap + j) * H + h) * D + c0;
  *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_decode_block_mean(const DecodeArgs& a, cudaStream_t s) {
  nsa_decode_block_mean_kernel<<<dim3(a.batch, a.geo.Hkv), a.geo.D / 8, 0, s>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ routing scores
// S[t, g, j] = sum over the G heads h of group g of q[t, h] . Kbar[j, g] for
// the blocks j < t / l' (the complete blocks before t's own block).
//
// One persistent CTA per SM walks dense tiles of 128 MMA rows = (128 / G)
// consecutive tokens x the G heads of one KV group (heaviest tiles first).
// Per chunk of 128 mean keys, one 128 x 128 tcgen05 product S^T = Kbar Q^T
// puts the keys on TMEM lanes and the (token, head) rows on columns, so a
// thread owns one key and sums each token's G columns in registers; a warp's
// stores of one token's scores are 128 consecutive bytes.
// Warp roles: 0 = TMA producer, 1 = tcgen05.mma issuer, 2..5 and 6..9 = two
// epilogue warpgroups that take alternate chunks.  TMEM holds four 128-column
// score buffers (chunk i of the CTA's sequence goes to buffer i % 4, owned by
// warpgroup i % 2), so the products run up to three chunks ahead of the
// epilogue.

namespace {

template <int D>
struct BsLayout {
  static constexpr int kStages = 4;
  static constexpr int kQBytes = kTileRows * D * 2;
  static constexpr int kChunkBytes = kChunk * D * 2;
  static constexpr int kQ = 0;                              // 2 buffers
  static constexpr int kRing = kQ + 2 * kQBytes;            // kStages
  static constexpr int kBars = kRing + kStages * kChunkBytes;
  static constexpr int kW = kBars + 32 * 8;                 // per epilogue warpgroup: a tile's
  static constexpr int kEnd = kW + 2 * kTileRows * 4;       // head weights [token][G] (fp32)
  // at least 116 KB so that one CTA owns an SM (it allocates all 512 TMEM columns)
  static constexpr int kSmem = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
};

constexpr int kBsThreads = 320;

struct BsItem {
  int valid, g, t0, T, row0, ntok, nc, blk0;
};

__device__ __forceinline__ BsItem bs_item(const PrefillArgs& a, int k) {
  BsItem it{};
  const int tiles = a.meta->tiles_total, H = a.geo.Hkv;
  if (k >= tiles * H) return it;
  it.valid = 1;
  const int tau = tiles - 1 - k / H;  // heaviest (latest) tiles first
  it.g = k % H;
  const int b = seq_of_offset(a.tile_off, a.batch, tau);
  it.t0 = (tau - a.tile_off[b]) * a.geo.tpt;
  const int c0 = __ldg(a.cu + b);
  it.T = __ldg(a.cu + b + 1) - c0;
  it.row0 = c0 + it.t0;
  it.ntok = min(a.geo.tpt, it.T - it.t0);
  // blocks before the own block of the tile's last token (token-level
  // selection: every token up to and including it)
  const int nb = a.token_select ? it.t0 + it.ntok : (it.t0 + it.ntok - 1) >> a.geo.lg_ls;
  it.nc = (nb + kChunk - 1) / kChunk;
  it.blk0 = a.cmp_off[b];
  return it;
}

// One chunk's epilogue for the thread owning key `key` (TMEM lane): the G
// columns of each token summed, stored where the key is a candidate of the
// token (key < t / l').  With token-level selection (`wts` non-null: the
// tile's head weights [token][G] in shared memory, zero past its tokens) the
// G columns of a token are indexer heads: the score is the sum of the
// token's head weights times ReLU(column), and keys up to and including the
// token take part.  The TMEM loads of 64 columns are issued before one wait.
template <int G>
__device__ __forceinline__ void bs_rows(uint32_t taddr, float* srow, size_t tok_stride, int key,
                                        int t0, int ntok, int lg_ls, bool live,
                                        const float* wts) {
#pragma unroll 1
  for (int g4 = 0; g4 < kTileRows / 64; ++g4) {
    float v[4][16];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld16(taddr + g4 * 64 + q * 16, v[q]);
    tmem_ld_wait();
#pragma unroll
    for (int kt = 0; kt < 64 / G; ++kt) {
      const int tok = (g4 * 64 + kt * G) / G;
      float s = 0.f;
      if (wts) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const int c = kt * G + j;
          s += wts[tok * G + j] * fmaxf(v[c >> 4][c & 15], 0.f);
        }
      } else {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const int c = kt * G + j;
          s += v[c >> 4][c & 15];
        }
      }
      const bool vis = wts ? key <= t0 + tok : key < ((t0 + tok) >> lg_ls);
      if (live && tok < ntok && vis) srow[(size_t)tok * tok_stride] = s;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kBsThreads, 1)
    nsa_block_score_kernel(const __grid_constant__ PrefillArgs a,
                           const __grid_constant__ PrefillMaps maps) {
  using L = BsLayout<D>;
  constexpr int KSTEPS = D / 16;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;    // [2]
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* st_full = bars + 4;   // [4]
  uint64_t* st_empty = bars + 8;  // [4]
  uint64_t* s_full = bars + 12;   // [4] TMEM score buffers
  uint64_t* s_empty = bars + 16;  // [4]
  uint64_t* fin = bars + 20;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 22);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);

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
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(st_full + i, 1);
      mbar_init(st_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, 4);
    }
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
      tma_prefetch_desc(&maps.kc);
      int qc = 0, sc = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const BsItem it = bs_item(a, k);
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
        for (int c = 0; c < it.nc; ++c) {
          const int s = sc % L::kStages, us = sc / L::kStages;
          if (us > 0 && !mbar_wait(st_empty + s, (us - 1) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            break;
          }
          uint8_t* dst = sm + L::kRing + s * L::kChunkBytes;
          mbar_arrive_expect_tx(st_full + s, L::kChunkBytes);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(dst + h * 16384, &maps.kc, st_full + s, h * 64, it.g, it.blk0 + c * kChunk);
          ++sc;
        }
      }
      // drain: every issued copy has landed before the CTA retires
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
      constexpr uint32_t id = idesc_bf16(128, 128, false, false);
      int qc = 0, sc = 0, cc = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const BsItem it = bs_item(a, k);
        if (!it.valid) break;
        if (it.nc == 0) continue;
        const int qb = qc & 1;
        if (!mbar_wait(q_full + qb, (qc >> 1) & 1, abort_flag, status, kWaitCycles)) break;
        for (int c = 0; c < it.nc; ++c, ++cc) {
          const int s = sc % L::kStages, buf = cc & 3, ub = cc >> 2;
          if (!mbar_wait(st_full + s, (sc / L::kStages) & 1, abort_flag, status, kWaitCycles) ||
              (ub > 0 && !mbar_wait(s_empty + buf, (ub - 1) & 1, abort_flag, status, kWaitCycles))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t A = sbase + L::kRing + s * L::kChunkBytes;
          const uint32_t B = sbase + L::kQ + qb * L::kQBytes;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_bf16_ss(tmem + buf * 128, smem_desc(A + off, 16, 1024, kLayoutSw128),
                        smem_desc(B + off, 16, 1024, kLayoutSw128), id, ks > 0);
          }
          mma_commit(st_empty + s);
          mma_commit(s_full + buf);
          ++sc;
        }
        if (!ok) break;
        mma_commit(q_empty + qb);
        ++qc;
      }
      mma_commit(fin);
      volatile int never = 0;
      mbar_wait(fin, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int w = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int Hkv = a.geo.Hkv, cap = a.geo.cmp_cap, lgG = a.geo.lg_G, lg_ls = a.geo.lg_ls;
    const size_t tok_stride = (size_t)Hkv * cap;
    float* wsm = reinterpret_cast<float*>(sm + L::kW) + w * kTileRows;
    int cc = 0, w_item = -1;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const BsItem it = bs_item(a, k);
      if (!it.valid) break;
      for (int c = 0; c < it.nc; ++c, ++cc) {
        if ((cc & 1) != w) continue;
        if (a.token_select && w_item != k) {
          // the tile's head weights, once per tile and warpgroup (named
          // barrier 1 + w over its 128 threads: the previous tile's reads are
          // done before the copy, the copy before the reads)
          asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
          wsm[r] = r < it.ntok * G ? __ldg(a.gates + (size_t)it.row0 * G + r) : 0.f;
          asm volatile("bar.sync %0, 128;" ::"r"(1 + w) : "memory");
          w_item = k;
        }
        const int buf = cc & 3, ub = cc >> 2;
        mbar_wait(s_full + buf, ub & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
        const int key = c * kChunk + r;
        float* srow = a.scores + ((size_t)it.row0 * Hkv + it.g) * cap + key;
        const bool live = !*abort_flag;
        const uint32_t taddr = lane_addr + buf * 128;
        // per-token indexer head weights of the tile (token-level selection)
        const float* wts = a.token_select ? wsm : nullptr;
        switch (lgG) {
          case 0: bs_rows<1>(taddr, srow, tok_stride, key, it.t0, it.ntok, lg_ls, live, wts); break;
          case 1: bs_rows<2>(taddr, srow, tok_stride, key, it.t0, it.ntok, lg_ls, live, wts); break;
          case 2: bs_rows<4>(taddr, srow, tok_stride, key, it.t0, it.ntok, lg_ls, live, wts); break;
          case 3: bs_rows<8>(taddr, srow, tok_stride, key, it.t0, it.ntok, lg_ls, live, wts); break;
          default: bs_rows<16>(taddr, srow, tok_stride, key, it.t0, it.ntok, lg_ls, live, wts); break;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty + buf);
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
cudaError_t launch_block_score_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                                 cudaStream_t s) {
  using L = BsLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_block_score_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = num_sms < kMaxPersistentCtas ? num_sms : kMaxPersistentCtas;
  nsa_block_score_kernel<D><<<grid, kBsThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_score(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                               cudaStream_t s) {
  return a.geo.D == 128 ? launch_block_score_t<128>(a, m, num_sms, s)
                        : launch_block_score_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
