// Small prefill kernels: per-call metadata and top-n block selection
// (step 4; block compression, step 1, is in k_compress.cu).
//
// Selection follows the config page, section 3 (select_top_k), and the
// manufacturing page, same section (the highest-scoring blocks are kept);
// the selection itself is in topn_util.cuh.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "topn_util.cuh"

namespace nsa {

// ------------------------------------------------------------------ metadata
// One thread scans cu_seqlens: compressed-row and tile offsets per sequence,
// and a consistency check (lengths within [0, max_seqlen], totals match).
__global__ void nsa_meta_kernel(PrefillArgs a, int max_seqlen) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int B = a.batch;
  int bad = (__ldg(a.cu) != 0);
  int c = 0, tl = 0;
  a.cmp_off[0] = 0;
  a.tile_off[0] = 0;
  for (int b = 0; b < B; ++b) {
    const int T = __ldg(a.cu + b + 1) - __ldg(a.cu + b);
    if (T < 0 || T > max_seqlen) {
      bad = 1;
      break;
    }
    c += num_cmp_blocks(T, a.geo.l, a.geo.d);
    tl += (T + a.geo.tpt - 1) / a.geo.tpt;
    a.cmp_off[b + 1] = c;
    a.tile_off[b + 1] = tl;
  }
  if (!bad && __ldg(a.cu + B) != a.total_tokens) bad = 1;
  a.meta->bad = bad;
  a.meta->cmp_total = bad ? 0 : c;
  a.meta->tiles_total = bad ? 0 : tl;
  if (bad) atomicCAS(a.status, 0, sm100::kDeviceBadInputCode);
}

cudaError_t launch_meta(const PrefillArgs& a, cudaStream_t s) {
  nsa_meta_kernel<<<1, 32, 0, s>>>(a, a.geo.max_seqlen);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ top-n
// One warp per (token, KV group); the selection itself is warp_topn.  With
// l == d == l' the candidates' scores are the compressed-block scores; else
// each selection block's score is first summed from the compressed blocks
// that overlap it (written to the selection-score table, then ranked).  In
// select-only block attention the scores are routing scores and the query's
// own block is always taken.
__global__ void __launch_bounds__(256) nsa_topn_kernel(PrefillArgs a) {
  if (a.meta->bad) return;
  __shared__ unsigned hist_all[8][256];
  __shared__ unsigned long long cand_all[8][kTopnCand];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int H = a.geo.Hkv, n = a.geo.n;
  const long long row = (long long)blockIdx.x * 8 + warp;
  if (row >= (long long)a.total_tokens * H) return;
  const int tg = (int)(row / H), g = (int)(row % H);
  const int b = seq_of_token(a.cu, a.batch, tg);
  const int t = tg - __ldg(a.cu + b);
  const float* S = a.scores + ((size_t)tg * H + g) * a.geo.cmp_cap;
  int* out = a.sel + ((size_t)tg * H + g) * n;
  auto put = [&](int i, int j) { out[i] = j; };
  if (a.select_only) {
    // select-only block attention: the n - 1 best of the complete blocks
    // before t's own block (routing scores), then the own block, which has
    // the largest index, last
    const int cur = t >> a.geo.lg_ls, m = n - 1;
    if (m > 0) {
      auto score = [&](int j) { return S[j]; };
      if (!(cur <= 1024 && m <= 32 && warp_topn_regs(score, cur, cur, m, cand_all[warp], put)))
        warp_topn(score, cur, cur, m, hist_all[warp], put);
    }
    __syncwarp();
    if (lane == 0) {
      const int taken = cur < m ? cur : m;
      out[taken] = cur;
      for (int i = taken + 1; i < n; ++i) out[i] = -1;
    }
    return;
  }
  const int ncmp = num_cmp_blocks(t + 1, a.geo.l, a.geo.d), ncand = t / a.geo.ls + 1;
  if (!a.geo.remap) {
    auto score = [&](int j) { return S[j]; };
    if (ncand <= 1024 && n <= 32 && warp_topn_regs(score, ncmp, ncand, n, cand_all[warp], put))
      return;
    warp_topn(score, ncmp, ncand, n, hist_all[warp], put);
    return;
  }
  float* Ssel = a.sel_scores + ((size_t)tg * H + g) * a.geo.sel_cap;
  for (int j = lane; j < ncand; j += 32)
    Ssel[j] = remap_score(a.geo, [&](int i) { return S[i]; }, ncmp, j);
  __syncwarp();
  auto score = [&](int j) { return Ssel[j]; };
  if (ncand <= 1024 && n <= 32 && warp_topn_regs(score, ncand, ncand, n, cand_all[warp], put))
    return;
  warp_topn(score, ncand, ncand, n, hist_all[warp], put);
}

cudaError_t launch_topn(const PrefillArgs& a, cudaStream_t s) {
  const long long rows = (long long)a.total_tokens * a.geo.Hkv;
  if (rows == 0) return cudaSuccess;
  nsa_topn_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ timeout self-test
// One CTA waits on an mbarrier that nothing will ever arrive on; the bounded
// wait gives up after `cycles` and records the timeout in the status word.
__global__ void nsa_timeout_selftest_kernel(int* status, long long cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, status, cycles);
}

cudaError_t launch_timeout_selftest(int* status, long long cycles, cudaStream_t s) {
  nsa_timeout_selftest_kernel<<<1, 32, 0, s>>>(status, cycles);
  return cudaGetLastError();
}

}  // namespace nsa
