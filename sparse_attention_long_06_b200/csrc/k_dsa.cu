// Token-level top-k attention (DSA style): selection and the attention over
// the selected tokens.
//
// "DeepSeek V3.2-Exp sparse attention" page (bjdmk.com.cn/news/5181035),
// sections 1 and 3: a light indexer with a ReLU scores every earlier token of
// a query and the top_k of them (2048 on the page) take part in the main
// attention.  The index scores come from the routing-score kernel in its
// token-level mode (k_bsel.cu); here each query's top_k tokens are selected
// (ties to the lower index) and every query head attends to the keys and
// values of its KV group at those tokens.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "topn_util.cuh"

namespace nsa {
using namespace sm100;

// ------------------------------------------------------------------ selection
// One warp per query token t: the top_k of its t + 1 index scores, ascending,
// -1 padded (the register path for rows of at most 1024 candidates and
// top_k <= 32, else the radix select).
__global__ void __launch_bounds__(256) nsa_token_topk_kernel(PrefillArgs a, int top_k) {
  if (a.meta->bad) return;
  __shared__ unsigned hist_all[8][256];
  __shared__ unsigned long long cand_all[8][kTopnCand];
  const int warp = threadIdx.x / 32;
  const long long tg = (long long)blockIdx.x * 8 + warp;
  if (tg >= a.total_tokens) return;
  const int b = seq_of_token(a.cu, a.batch, (int)tg);
  const int t = (int)tg - __ldg(a.cu + b);
  const float* S = a.scores + (size_t)tg * a.geo.cmp_cap;
  int* out = a.sel + (size_t)tg * top_k;
  auto put = [&](int i, int j) { out[i] = j; };
  auto score = [&](int j) { return S[j]; };
  const int ncand = t + 1;
  if (ncand <= 1024 && top_k <= 32 && warp_topn_regs(score, ncand, ncand, top_k, cand_all[warp], put))
    return;
  warp_topn(score, ncand, ncand, top_k, hist_all[warp], put);
}

// ------------------------------------------------------------------ attention
// One CTA per query token, one warp per KV group: the group's G <= 16 heads
// are the 16 rows of mma.sync m16n8k16 bf16 products with fp32 accumulators
// (rows past G are zero queries whose results are dropped).  The selected
// tokens are taken 32 at a time; their keys and values for every group are
// copied (16-byte cp.async, double buffered) into shared memory rows padded
// to D + 8 elements, so that the eight rows an operand fragment spans fall
// in different banks.  Per step and warp: S = Q K^T (queries as A fragments
// kept in registers, keys read as B fragments), an online softmax on the
// accumulator fragments (row statistics over the four threads of a quad),
// then O += P V with P re-packed from the S fragments as A fragments and V
// read by ldmatrix.trans.
namespace {

constexpr int kDsaKeys = 32;  // selected tokens per step

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

template <int D, int HKV>
__global__ void __launch_bounds__(HKV * 32) nsa_token_attn_kernel(PrefillArgs a, int top_k) {
  if (a.meta->bad) return;
  constexpr int RS = D + 8;                         // padded row, elements
  constexpr int kRows = HKV * kDsaKeys;             // rows of one step
  constexpr int kBufBytes = kRows * RS * 2;         // keys (or values) of one step
  constexpr int KS = D / 16;                        // k-steps of q . k
  constexpr int NT = D / 8;                         // n-tiles of O
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* kbuf = sm;                               // [2][HKV][keys][RS]
  uint8_t* vbuf = sm + 2 * kBufBytes;               // [2][HKV][keys][RS]
  int* idx = reinterpret_cast<int*>(sm + 4 * kBufBytes);  // [2][keys]
  const int Hq = a.geo.Hq, G = Hq / HKV;
  const int tg = blockIdx.x;
  if (tg >= a.total_tokens) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane >> 2, tig = lane & 3;
  const int b = seq_of_token(a.cu, a.batch, tg);
  const int t = tg - __ldg(a.cu + b);
  const int cu0 = __ldg(a.cu + b);
  const int nsel = min(top_k, t + 1);
  const int* sel = a.sel + (size_t)tg * top_k;
  const int g = warp;  // this warp's KV group

  // query A fragments: rows gid and gid + 8 (heads of the group), k-step ks
  uint32_t qa[KS][4];
  {
    const uint16_t* qg = a.q + ((size_t)tg * Hq + (size_t)g * G) * D;
    auto ld = [&](int row, int col) -> uint32_t {
      return row < G ? __ldg(reinterpret_cast<const uint32_t*>(qg + (size_t)row * D + col)) : 0u;
    };
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = ld(gid, ks * 16 + tig * 2);
      qa[ks][1] = ld(gid + 8, ks * 16 + tig * 2);
      qa[ks][2] = ld(gid, ks * 16 + tig * 2 + 8);
      qa[ks][3] = ld(gid + 8, ks * 16 + tig * 2 + 8);
    }
  }
  const int nsteps = (nsel + kDsaKeys - 1) / kDsaKeys;
  auto issue = [&](int step) {
    const int buf = step & 1;
    if (threadIdx.x < kDsaKeys) {
      const int i = step * kDsaKeys + threadIdx.x;
      idx[buf * kDsaKeys + threadIdx.x] = i < nsel ? __ldg(sel + i) : -1;
    }
    const uint32_t kb = smem_u32(kbuf + buf * kBufBytes), vb = smem_u32(vbuf + buf * kBufBytes);
    for (int e = threadIdx.x; e < kRows * (D / 8); e += HKV * 32) {
      const int c8 = e % (D / 8), row = e / (D / 8);  // row = group * keys + key
      const int key = row % kDsaKeys, gg = row / kDsaKeys;
      const int i = step * kDsaKeys + key;
      const int s = i < nsel ? __ldg(sel + i) : -1;
      const bool ok = s >= 0;
      const size_t src = ((size_t)(cu0 + (ok ? s : 0)) * HKV + gg) * D + c8 * 8;
      cp_async16(kb + (row * RS + c8 * 8) * 2, a.k + src, ok);
      cp_async16(vb + (row * RS + c8 * 8) * 2, a.v + src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[n][c] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows gid, gid + 8
  const float sl2 = a.geo.scale_log2;
  if (nsteps > 0) issue(0);
  for (int step = 0; step < nsteps; ++step) {
    const int buf = step & 1;
    if (step + 1 < nsteps) {
      issue(step + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint16_t* kr = reinterpret_cast<const uint16_t*>(kbuf + buf * kBufBytes) + (size_t)g * kDsaKeys * RS;
    const uint32_t vaddr = smem_u32(vbuf + buf * kBufBytes) + (uint32_t)(g * kDsaKeys * RS * 2);
    // S = Q K^T: four n-tiles of 8 keys
    float sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) sacc[nt][c] = 0.f;
      const uint16_t* krow = kr + (size_t)(nt * 8 + gid) * RS;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(krow + ks * 16 + tig * 2);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(krow + ks * 16 + tig * 2 + 8);
        mma_bf16_16816(sacc[nt], qa[ks], b0, b1);
      }
    }
    // online softmax; columns (keys) of this thread: nt * 8 + tig * 2 + {0, 1}
    float mloc[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = nt * 8 + tig * 2 + (c & 1);
        const bool on = idx[buf * kDsaKeys + key] >= 0;
        sacc[nt][c] = on ? sacc[nt][c] * sl2 : -INFINITY;
        mloc[c >> 1] = fmaxf(mloc[c >> 1], sacc[nt][c]);
      }
    }
    float f[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mloc[r] = fmaxf(mloc[r], __shfl_xor_sync(0xffffffffu, mloc[r], 1));
      mloc[r] = fmaxf(mloc[r], __shfl_xor_sync(0xffffffffu, mloc[r], 2));
      const float mn = fmaxf(m_run[r], mloc[r]);
      f[r] = (m_run[r] == -INFINITY) ? 0.f : ex2(m_run[r] - mn);
      m_run[r] = mn;
    }
    float lsum[2] = {0.f, 0.f};
    uint32_t pa[2][4];  // P as A fragments of the two k-steps (16 keys each)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      float p[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float mr = m_run[c >> 1];
        p[c] = (mr == -INFINITY || sacc[nt][c] == -INFINITY) ? 0.f : ex2(sacc[nt][c] - mr);
        lsum[c >> 1] += p[c];
      }
      const uint32_t lo = pack_bf16x2(p[0], p[1]), hi = pack_bf16x2(p[2], p[3]);
      pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
      pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 1);
      lsum[r] += __shfl_xor_sync(0xffffffffu, lsum[r], 2);
      l_run[r] = l_run[r] * f[r] + lsum[r];
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= f[0];
      o[n][1] *= f[0];
      o[n][2] *= f[1];
      o[n][3] *= f[1];
    }
    // O += P V: k-steps of 16 keys, n-tiles of 8 channels; V rows by ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      // lanes 0-7 address keys kk*16 + 0..7, lanes 8-15 keys kk*16 + 8..15
      const int vrow = kk * 16 + (lane & 15);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint32_t b0, b1;
        ldmatrix_x2_trans(b0, b1, vaddr + (uint32_t)((vrow * RS + n * 8) * 2));
        mma_bf16_16816(o[n], pa[kk], b0, b1);
      }
    }
    __syncthreads();  // the buffer is refilled two steps on
  }
  // rows gid and gid + 8 of the group: heads g * G + row
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = gid + r * 8;
    if (row >= G) continue;
    const float inv = l_run[r] > 0.f ? 1.f / l_run[r] : 0.f;
    const size_t base = ((size_t)tg * Hq + (size_t)g * G + row) * D;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = n * 8 + tig * 2;
      const float v0 = o[n][r * 2] * inv, v1 = o[n][r * 2 + 1] * inv;
      if (a.geo.out_f32) {
        *reinterpret_cast<float2*>(static_cast<float*>(a.out) + base + col) = make_float2(v0, v1);
      } else {
        *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.out) + base + col) = pack_bf16x2(v0, v1);
      }
    }
  }
}

template <int D, int HKV>
cudaError_t launch_token_attn_t(const PrefillArgs& a, int top_k, cudaStream_t s) {
  constexpr int RS = D + 8;
  const size_t smem = 4 * (size_t)HKV * kDsaKeys * RS * 2 + 2 * kDsaKeys * 4;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_token_attn_kernel<D, HKV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  nsa_token_attn_kernel<D, HKV><<<a.total_tokens, HKV * 32, smem, s>>>(a, top_k);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_token_topk(const PrefillArgs& a, int top_k, cudaStream_t s) {
  if (a.total_tokens <= 0) return cudaSuccess;
  nsa_token_topk_kernel<<<(unsigned)((a.total_tokens + 7) / 8), 256, 0, s>>>(a, top_k);
  return cudaGetLastError();
}

// a.geo here is the main attention's geometry (Hq, Hkv, D, scale, output)
cudaError_t launch_token_attn(const PrefillArgs& a, int top_k, cudaStream_t s) {
  if (a.total_tokens <= 0) return cudaSuccess;
  const int H = a.geo.Hkv;
  if (a.geo.D == 128) {
    switch (H) {
      case 1: return launch_token_attn_t<128, 1>(a, top_k, s);
      case 2: return launch_token_attn_t<128, 2>(a, top_k, s);
      case 4: return launch_token_attn_t<128, 4>(a, top_k, s);
      default: return launch_token_attn_t<128, 8>(a, top_k, s);
    }
  }
  switch (H) {
    case 1: return launch_token_attn_t<64, 1>(a, top_k, s);
    case 2: return launch_token_attn_t<64, 2>(a, top_k, s);
    case 4: return launch_token_attn_t<64, 4>(a, top_k, s);
    default: return launch_token_attn_t<64, 8>(a, top_k, s);
  }
}

}  // namespace nsa
