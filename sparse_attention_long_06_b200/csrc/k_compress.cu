// Block compression (step 1) on the tensor cores.
//
// "DeepSeek NSA config.toml" page, section 3 (compress_block_size) and
// "DeepSeek NSA in manufacturing" page, section on what dynamic sparsity
// sparsifies: each block of l keys (values) is flattened and mapped by one
// learned linear layer to a single compressed token:
//   Kc[r, h, c] = sum_{p < l, c' < D} W[h, c, p D + c'] X[tok0(r) + p, h, c']
// for every complete block r of every sequence (tok0 = the sequence start
// plus d times the block's index in it).
//
// Per (tensor, head) this is a GEMM [blocks x l D] x [l D x D].  The fp32
// weights are split exactly into three bf16 terms, W = hi + mid + lo (each
// term holds the next 8 of fp32's 24 significand bits), so every product of
// a bf16 key with a term is exact and the tcgen05 products accumulate in
// fp32: the result is the fp32 sum of the exact products, as in a plain fp32
// GEMM, computed on the tensor cores.
//
// Tiles: 128 blocks (MMA rows, one per TMEM lane) x 64 output channels.  The
// K dimension runs over 64-channel chunks of one token offset p.  The A tile
// of a chunk (128 rows of 128 contiguous bytes) starts at a row that depends
// on each block's sequence, so four producer warps load it with cp.async
// (thread = row) into the 128-byte-swizzled K-major layout; the three B tiles
// (64 weight rows x 64 k of each term) come by TMA.  Warp 4 issues the
// products.  The tensor cores' fp32 accumulation is not rounded to nearest at
// every step, and over the 1536 products of a row (l D / 16 k-steps x 3
// terms) its error reached 1e-5 relative; so each group of four chunks (48
// product steps) starts a fresh accumulator in one of eight rotating TMEM
// buffers, and four drain warps (5-8) add the group sums in fp32 registers
// and store the bf16 row.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"

namespace nsa {
using namespace sm100;

// ------------------------------------------------------------------ weight split
// planes [tensor][term][Hkv][D][l D] bf16 from W_K, W_V [Hkv][D][l D] fp32:
// hi = rn(w), mid = rn(w - hi), lo = rn(w - hi - mid).  The differences are
// exact in fp32 and the last one fits 8 significand bits, so hi + mid + lo = w.
__global__ void __launch_bounds__(256) nsa_weight_split_kernel(const float* w_k, const float* w_v,
                                                               uint16_t* planes, long long per) {
  const long long i4 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i4 >= 2 * per) return;
  const int z = i4 >= per ? 1 : 0;
  const long long i = i4 - z * per;
  const float4 w = __ldg(reinterpret_cast<const float4*>((z ? w_v : w_k) + i));
  const float x[4] = {w.x, w.y, w.z, w.w};
  uint16_t t[3][4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat16 hi = __float2bfloat16_rn(x[e]);
    const float r1 = x[e] - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    t[0][e] = *reinterpret_cast<const uint16_t*>(&hi);
    t[1][e] = *reinterpret_cast<const uint16_t*>(&mid);
    t[2][e] = *reinterpret_cast<const uint16_t*>(&lo);
  }
#pragma unroll
  for (int term = 0; term < 3; ++term) {
    uint16_t* dst = planes + ((long long)z * 3 + term) * per + i;
    *reinterpret_cast<uint2*>(dst) =
        make_uint2((uint32_t)t[term][0] | ((uint32_t)t[term][1] << 16),
                   (uint32_t)t[term][2] | ((uint32_t)t[term][3] << 16));
  }
}

namespace {

struct CpLayout {
  static constexpr int kStages = 4;
  static constexpr int kABytes = 128 * 128;  // 128 rows x 64 channels
  static constexpr int kBBytes = 64 * 128;   // 64 weight rows x 64 k, one term
  static constexpr int kStageBytes = kABytes + 3 * kBBytes;
  static constexpr int kBars = kStages * kStageBytes;
  static constexpr int kEnd = kBars + 32 * 8;
  static constexpr int kSmem = kEnd;
  static_assert(kStageBytes % 1024 == 0, "swizzled tiles stay 1024-byte aligned");
};

constexpr int kCpThreads = 288;  // warps 0-3 A rows, warp 4 products, warps 5-8 drain
constexpr int kCpDepth = 3;      // cp.async chunks in flight per producer thread
constexpr int kCpGroup = 4;      // chunks per accumulator group
constexpr int kCpBufs = 8;       // TMEM accumulators of 64 columns

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct CpItem {
  int valid, z, h, nh, m0;
};

// Items in row-tile-major order, so that the CTAs sharing an A tile (the
// D / 64 output halves) run together and the second read hits L2.
__device__ __forceinline__ CpItem cp_item(const PrefillArgs& a, int k, int nhalves) {
  CpItem it{};
  const int H = a.geo.Hkv;
  const int per_tile = 2 * H * nhalves;
  const int tiles = (a.cmp_rows + 127) / 128;
  if (k >= tiles * per_tile) return it;
  it.valid = 1;
  it.m0 = (k / per_tile) * 128;
  const int rem = k % per_tile;
  it.z = rem / (H * nhalves);
  it.h = (rem / nhalves) % H;
  it.nh = rem % nhalves;
  return it;
}

template <int D>
__global__ void __launch_bounds__(kCpThreads, 1)
    nsa_compress_tc_kernel(const __grid_constant__ PrefillArgs a,
                           const __grid_constant__ PrefillMaps maps) {
  using L = CpLayout;
  constexpr int NH = D / 64;  // 64-channel halves of a row
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* full = bars + 0;        // [4] A rows (128 arrivals) + B terms (tx)
  uint64_t* empty = bars + 4;       // [4] products done with the stage
  uint64_t* acc_full = bars + 8;    // [8] a group's sum complete in its buffer
  uint64_t* acc_empty = bars + 16;  // [8] the buffer read by the drain warps
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 24);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 25);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (a.meta->bad) return;
  if (smem_u32(sm) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDeviceTimeoutCode);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(full + i, 129);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < kCpBufs; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 64 * kCpBufs);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  int* status = a.status;
  const int H = a.geo.Hkv, l = a.geo.l;
  const int nk = l * NH;  // 64-channel chunks of the K dimension
  const int C = a.meta->cmp_total;

  if (warp < 4) {
    // ------------------------------------------------------------ rows: A tiles
    const int i = threadIdx.x;  // row of the tile
    const uint32_t arow = (i >> 3) * 1024 + (i & 7) * 128;
    int it_chunk = 0;
    bool ok = true;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const CpItem it = cp_item(a, k, NH);
      if (!it.valid) break;
      const int r = it.m0 + i;
      const bool live = r < C;
      long long tok0 = 0;
      if (live) {
        const int b = seq_of_offset(a.cmp_off, a.batch, r);
        tok0 = __ldg(a.cu + b) + (long long)(r - a.cmp_off[b]) * a.geo.d;
      }
      const uint16_t* X = it.z ? a.v : a.k;
      const uint16_t* src_row = X + ((size_t)tok0 * H + it.h) * D;
      int pending = 0;  // chunks issued whose arrival is still owed
      for (int kc = 0; kc < nk; ++kc, ++it_chunk) {
        const int s = it_chunk % L::kStages, u = it_chunk / L::kStages;
        if (ok && u > 0 && !mbar_wait(empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles))
          ok = false;
        uint8_t* stage = sm + s * L::kStageBytes;
        if (i == 0) {
          mbar_arrive_expect_tx(full + s, 3 * L::kBBytes);
          if (ok) {
#pragma unroll
            for (int term = 0; term < 3; ++term)
              tma_load_2d(stage + L::kABytes + term * L::kBBytes, &maps.wpl, full + s, kc * 64,
                          ((it.z * 3 + term) * H + it.h) * D + it.nh * 64);
          }
        }
        const int p = kc / NH, half = kc % NH;
        const uint16_t* src = src_row + (size_t)p * H * D + half * 64;
        const uint32_t dst = sbase + s * L::kStageBytes + arow;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16(dst + ((j ^ (i & 7)) << 4), live ? src + j * 8 : a.k, live && ok);
        cp_async_commit();
        ++pending;
        if (pending == kCpDepth) {
          // the oldest chunk in flight has landed: publish it to the products
          cp_async_wait<kCpDepth - 1>();
          fence_async_smem();
          mbar_arrive(full + (it_chunk - (kCpDepth - 1)) % L::kStages);
          --pending;
        }
      }
      cp_async_wait<0>();
      fence_async_smem();
      for (int q = pending; q > 0; --q) mbar_arrive(full + (it_chunk - q) % L::kStages);
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ products
    if (lane == 0) {
      constexpr uint32_t id = idesc_bf16(128, 64, false, false);
      int it_chunk = 0, grp = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok; k += gridDim.x) {
        const CpItem it = cp_item(a, k, NH);
        if (!it.valid) break;
        for (int kc = 0; kc < nk; ++kc, ++it_chunk) {
          const int s = it_chunk % L::kStages;
          const int buf = grp % kCpBufs, ub = grp / kCpBufs;
          if (kc % kCpGroup == 0 && ub > 0 &&
              !mbar_wait(acc_empty + buf, (ub - 1) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            break;
          }
          if (!mbar_wait(full + s, (it_chunk / L::kStages) & 1, abort_flag, status, kWaitCycles)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t A = sbase + s * L::kStageBytes;
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint32_t B = A + L::kABytes + term * L::kBBytes;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16_ss(tmem + buf * 64, smem_desc(A + ks * 32, 16, 1024, kLayoutSw128),
                          smem_desc(B + ks * 32, 16, 1024, kLayoutSw128), id,
                          (kc % kCpGroup != 0 || term > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(empty + s);
          if (kc % kCpGroup == kCpGroup - 1) {
            mma_commit(acc_full + buf);
            ++grp;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ drain: group sums, bf16 rows
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // TMEM lane quadrant of this warp
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    int grp = 0;
    for (int k = blockIdx.x;; k += gridDim.x) {
      const CpItem it = cp_item(a, k, NH);
      if (!it.valid) break;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      for (int g = 0; g < nk / kCpGroup; ++g, ++grp) {
        const int buf = grp % kCpBufs, ub = grp / kCpBufs;
        mbar_wait(acc_full + buf, ub & 1, abort_flag, status, kWaitCycles);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t16[16];
          tmem_ld16(lane_addr + buf * 64 + c * 16, t16);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[c * 16 + j] += t16[j];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + buf);
      }
      const int r = it.m0 + row;
      if (r < a.cmp_rows && !*abort_flag) {
        uint16_t* out = (it.z ? a.v_cmp : a.k_cmp) + ((size_t)r * H + it.h) * D + it.nh * 64;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 w4 = make_uint4(pack_bf16x2(acc[8 * j], acc[8 * j + 1]),
                                      pack_bf16x2(acc[8 * j + 2], acc[8 * j + 3]),
                                      pack_bf16x2(acc[8 * j + 4], acc[8 * j + 5]),
                                      pack_bf16x2(acc[8 * j + 6], acc[8 * j + 7]));
          *reinterpret_cast<uint4*>(out + 8 * j) = w4;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 64 * kCpBufs);
  }
}

template <int D>
cudaError_t launch_compress_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                              cudaStream_t s) {
  using L = CpLayout;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_compress_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int items = ((a.cmp_rows + 127) / 128) * 2 * a.geo.Hkv * (D / 64);
  const int grid = items < num_sms ? items : num_sms;
  nsa_compress_tc_kernel<D><<<grid, kCpThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_weight_split(const PrefillArgs& a, uint16_t* planes, cudaStream_t s) {
  const long long per = (long long)a.geo.Hkv * a.geo.D * a.geo.l * a.geo.D;
  const long long threads = 2 * per / 4;
  nsa_weight_split_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(a.w_k, a.w_v, planes,
                                                                            per);
  return cudaGetLastError();
}

cudaError_t launch_compress_tc(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                               cudaStream_t s) {
  if (a.cmp_rows <= 0) return cudaSuccess;
  return a.geo.D == 128 ? launch_compress_t<128>(a, m, num_sms, s)
                        : launch_compress_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
