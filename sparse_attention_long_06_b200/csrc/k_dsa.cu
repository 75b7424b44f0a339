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
// One CTA per query token, eight warps.  The selected tokens are taken 32 at
// a time: their keys and values for every KV group are copied (16-byte
// cp.async, double buffered) into shared memory, keys as [group][8 channels]
// [token] so that lane = token reads without bank conflicts, values as
// [group][token][D].  Warp w owns heads w, w + 8, ...: per head, lane = token
// for q . k (q broadcast from shared memory), an online softmax over the
// warp, then lane = 4 channels for P V (probabilities broadcast by shuffle).
// fp32 throughout on the CUDA cores.
namespace {

constexpr int kDsaThreads = 256;
constexpr int kDsaKeys = 32;  // selected tokens per step

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

template <int D, int HKV>
__global__ void __launch_bounds__(kDsaThreads) nsa_token_attn_kernel(PrefillArgs a, int top_k) {
  if (a.meta->bad) return;
  constexpr int C8 = D / 8;                        // 16-byte pieces of a row
  constexpr int kKBytes = HKV * C8 * kDsaKeys * 16;  // keys of one step
  constexpr int kVBytes = HKV * kDsaKeys * D * 2;    // values of one step
  extern __shared__ __align__(16) uint8_t sm[];
  const int Hq = a.geo.Hq, G = Hq / HKV;
  uint8_t* kbuf = sm;                           // [2][HKV][C8][keys] uint4
  uint8_t* vbuf = sm + 2 * kKBytes;             // [2][HKV][keys][D] bf16
  uint16_t* qs = reinterpret_cast<uint16_t*>(sm + 2 * kKBytes + 2 * kVBytes);  // [Hq][D]
  int* idx = reinterpret_cast<int*>(qs + Hq * D);                               // [2][keys]

  const int tg = blockIdx.x;
  if (tg >= a.total_tokens) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = seq_of_token(a.cu, a.batch, tg);
  const int t = tg - __ldg(a.cu + b);
  const int cu0 = __ldg(a.cu + b);
  const int nsel = min(top_k, t + 1);  // selected tokens (the rest of the row is -1)
  const int* sel = a.sel + (size_t)tg * top_k;
  // the query rows of this token
  for (int i = threadIdx.x; i < Hq * C8; i += kDsaThreads)
    reinterpret_cast<uint4*>(qs)[i] = __ldg(reinterpret_cast<const uint4*>(a.q + (size_t)tg * Hq * D) + i);

  const int nsteps = (nsel + kDsaKeys - 1) / kDsaKeys;
  auto issue = [&](int step) {
    const int buf = step & 1;
    if (threadIdx.x < kDsaKeys) {
      const int i = step * kDsaKeys + threadIdx.x;
      idx[buf * kDsaKeys + threadIdx.x] = i < nsel ? __ldg(sel + i) : -1;
    }
    // each (group, key, piece) copy: keys and values
    const uint32_t kb = smem_u32(kbuf + buf * kKBytes), vb = smem_u32(vbuf + buf * kVBytes);
    for (int e = threadIdx.x; e < HKV * kDsaKeys * C8; e += kDsaThreads) {
      const int c8 = e % C8, key = (e / C8) % kDsaKeys, g = e / (C8 * kDsaKeys);
      const int i = step * kDsaKeys + key;
      const int s = i < nsel ? __ldg(sel + i) : -1;
      const bool ok = s >= 0;
      const size_t row = ((size_t)(cu0 + (ok ? s : 0)) * HKV + g) * D + c8 * 8;
      cp_async16(kb + ((g * C8 + c8) * kDsaKeys + key) * 16, a.k + row, ok);
      cp_async16(vb + ((g * kDsaKeys + key) * D + c8 * 8) * 2, a.v + row, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // per head of this warp: running maximum, sum and the lane's 4 (or 2)
  // output channels
  constexpr int kHeadsPerWarp = 64 / (kDsaThreads / 32);  // up to 64 heads
  constexpr int CPL = D / 32;                             // channels per lane
  float m_run[kHeadsPerWarp], l_run[kHeadsPerWarp], o[kHeadsPerWarp][CPL];
#pragma unroll
  for (int i = 0; i < kHeadsPerWarp; ++i) {
    m_run[i] = -INFINITY;
    l_run[i] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[i][c] = 0.f;
  }
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
    const uint4* kk = reinterpret_cast<const uint4*>(kbuf + buf * kKBytes);
    const uint16_t* vv = reinterpret_cast<const uint16_t*>(vbuf + buf * kVBytes);
    const bool on = idx[buf * kDsaKeys + lane] >= 0;
#pragma unroll
    for (int i = 0; i < kHeadsPerWarp; ++i) {
      const int h = warp + i * (kDsaThreads / 32);
      if (h >= Hq) break;
      const int g = h / G;
      // s = q_h . k_lane
      float s = 0.f;
      const uint16_t* qh = qs + h * D;
#pragma unroll 4
      for (int c8 = 0; c8 < C8; ++c8) {
        const uint4 kv = kk[(g * C8 + c8) * kDsaKeys + lane];
        const uint4 qv = *reinterpret_cast<const uint4*>(qh + c8 * 8);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = fmaf(__uint_as_float(qw[e] << 16), __uint_as_float(kw[e] << 16), s);
          s = fmaf(__uint_as_float(qw[e] & 0xFFFF0000u), __uint_as_float(kw[e] & 0xFFFF0000u), s);
        }
      }
      const float z = on ? s * sl2 : -INFINITY;
      float mz = z;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, off));
      const float mn = fmaxf(m_run[i], mz);
      const float p = on ? ex2(z - mn) : 0.f;
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      const float f = m_run[i] == -INFINITY ? 0.f : ex2(m_run[i] - mn);
      l_run[i] = l_run[i] * f + ps;
      m_run[i] = mn;
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[i][c] *= f;
      // O += p V: lane owns channels [lane * CPL, lane * CPL + CPL)
      for (int key = 0; key < kDsaKeys; ++key) {
        const float pk = __shfl_sync(0xffffffffu, p, key);
        const uint16_t* vr = vv + (g * kDsaKeys + key) * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[i][c] = fmaf(pk, __uint_as_float((uint32_t)vr[c] << 16), o[i][c]);
      }
    }
    __syncthreads();  // the buffer is refilled two steps on
  }
  // output rows
#pragma unroll
  for (int i = 0; i < kHeadsPerWarp; ++i) {
    const int h = warp + i * (kDsaThreads / 32);
    if (h >= Hq) break;
    const float inv = l_run[i] > 0.f ? 1.f / l_run[i] : 0.f;
    const size_t oi = ((size_t)tg * Hq + h) * D + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const float val = o[i][c] * inv;
      if (a.geo.out_f32) {
        static_cast<float*>(a.out)[oi + c] = val;
      } else {
        const __nv_bfloat16 bv = __float2bfloat16_rn(val);
        static_cast<uint16_t*>(a.out)[oi + c] = *reinterpret_cast<const uint16_t*>(&bv);
      }
    }
  }
}

template <int D, int HKV>
cudaError_t launch_token_attn_t(const PrefillArgs& a, int top_k, cudaStream_t s) {
  constexpr int C8 = D / 8;
  const size_t smem = 2 * (size_t)HKV * C8 * kDsaKeys * 16 + 2 * (size_t)HKV * kDsaKeys * D * 2 +
                      (size_t)a.geo.Hq * D * 2 + 2 * kDsaKeys * 4;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_token_attn_kernel<D, HKV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  nsa_token_attn_kernel<D, HKV><<<a.total_tokens, kDsaThreads, smem, s>>>(a, top_k);
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
