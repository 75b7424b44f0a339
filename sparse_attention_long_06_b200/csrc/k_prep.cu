// Small prefill kernels: per-call metadata, block compression (step 1) and
// top-n block selection (step 4).
//
// Compression follows the NSA pages: "DeepSeek NSA config.toml" page,
// section 3 (compress_block_size) and "DeepSeek NSA in manufacturing" page,
// section on what dynamic sparsity sparsifies (each block is flattened and
// mapped by one learned linear layer to a single compressed token).
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

// ------------------------------------------------------------------ compression
// Kc[r, h, c] = sum_{p < l, c' < D} W[h, c, p*D + c'] * X[tok0(r) + p, h, c']
// for every complete block r of every sequence (tok0 = first token of the
// block: the sequence start plus d times the block's index in it).  A tiled fp32 GEMM: CTA tile 32 blocks x D outputs, k-step 32.
// Rows in [cmp_total, cmp_rows) are zero-filled so that later tiles reading
// past the last sequence see finite values.
template <int D>
__global__ void __launch_bounds__(256) nsa_compress_kernel(PrefillArgs a) {
  if (a.meta->bad) return;
  constexpr int BM = 32, BK = 32, TN = D / 32;
  const int l = a.geo.l, H = a.geo.Hkv;
  const int h = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const uint16_t* X = is_v ? a.v : a.k;
  const float* W = (is_v ? a.w_v : a.w_k) + (size_t)h * D * l * D;
  uint16_t* out = is_v ? a.v_cmp : a.k_cmp;
  const int C = a.meta->cmp_total;
  const int r0 = blockIdx.x * BM;
  if (r0 >= a.cmp_rows) return;

  __shared__ int tok0[BM];
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][D + 4];
  const int tid = threadIdx.x;
  if (tid < BM) {
    const int r = r0 + tid;
    int t0 = -1;
    if (r < C) {
      const int b = seq_of_offset(a.cmp_off, a.batch, r);
      t0 = __ldg(a.cu + b) + (r - a.cmp_off[b]) * a.geo.d;
    }
    tok0[tid] = t0;
  }
  __syncthreads();

  const int ty = tid / 32, tx = tid % 32;  // rows ty*4..+4, cols tx*TN..+TN
  float acc[4][TN];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  const int K = l * D;
  for (int k0 = 0; k0 < K; k0 += BK) {
    const int p = k0 / D, c0 = k0 % D;
    {  // A tile: 32 rows x 32 k, 4 consecutive k per thread
      const int row = tid / 8, kk = (tid % 8) * 4;
      const int t0 = tok0[row];
      float v4[4] = {0.f, 0.f, 0.f, 0.f};
      if (t0 >= 0) {
        const uint2 raw = *reinterpret_cast<const uint2*>(X + ((size_t)(t0 + p) * H + h) * D + c0 + kk);
        v4[0] = __uint_as_float(raw.x << 16);
        v4[1] = __uint_as_float(raw.x & 0xFFFF0000u);
        v4[2] = __uint_as_float(raw.y << 16);
        v4[3] = __uint_as_float(raw.y & 0xFFFF0000u);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) As[kk + j][row] = v4[j];
    }
#pragma unroll
    for (int it = 0; it < D * BK / 4 / 256; ++it) {  // W tile: D rows x 32 k
      const int idx = it * 256 + tid;
      const int c = idx / 8, kq = (idx % 8) * 4;
      const float4 w4 = __ldg(reinterpret_cast<const float4*>(W + (size_t)c * K + k0 + kq));
      Ws[kq + 0][c] = w4.x;
      Ws[kq + 1][c] = w4.y;
      Ws[kq + 2][c] = w4.z;
      Ws[kq + 3][c] = w4.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[TN];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < TN; ++j) bv[j] = Ws[kk][tx * TN + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    if (r >= a.cmp_rows) continue;
    const bool live = r < C;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const __nv_bfloat16 bv = __float2bfloat16_rn(live ? acc[i][j] : 0.f);
      out[((size_t)r * H + h) * D + tx * TN + j] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
}

cudaError_t launch_compress(const PrefillArgs& a, cudaStream_t s) {
  if (a.cmp_rows <= 0) return cudaSuccess;
  dim3 grid((a.cmp_rows + 31) / 32, a.geo.Hkv, 2);
  if (a.geo.D == 128)
    nsa_compress_kernel<128><<<grid, 256, 0, s>>>(a);
  else
    nsa_compress_kernel<64><<<grid, 256, 0, s>>>(a);
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
