// Internal structures shared by the host API (nsa_api.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/nsa.h"

namespace nsa {

// Tokens of one dense tile: 128 MMA rows = (128 / G) tokens x G heads.
constexpr int kTileRows = 128;
// Keys per MMA chunk (M of the swap-AB products, N of the dense ones).
constexpr int kChunk = 128;
// Upper bound on persistent CTAs (grids are min(SM count, this)).
constexpr int kMaxPersistentCtas = 256;
// Header of every workspace: status word and counters.
constexpr size_t kHeaderBytes = 256;

struct Geometry {
  int D;        // head dim
  int Hq, Hkv;  // heads
  int G;        // Hq / Hkv
  int lg_G;     // log2(G)
  int tpt;      // tokens per dense tile = 128 / G
  int l;        // compression block length
  int d;        // compression stride (d <= l, l % d == 0)
  int ls;       // selection block length l'
  int lg_ls;    // log2(l')
  int remap;    // 1 unless l == d == l': selection scores are sums over the
                // compressed blocks that overlap each selection block
  int n;        // top-n
  int w;        // window
  int cmp_cap;  // row stride of the score table: compressed blocks of the
                // longest sequence, (max_seqlen - l) / d + 1
  int sel_cap;  // row stride of the selection-score table, max_seqlen / l' + 1
  int max_seqlen;
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  int out_f32;       // output dtype
};

// Per-call device metadata derived from cu_seqlens by nsa_meta_kernel.
struct Meta {
  int bad;          // nonzero when cu_seqlens is inconsistent (all kernels skip)
  int cmp_total;    // sum_b floor(T_b / l)
  int tiles_total;  // sum_b ceil(T_b / tpt)
  int pad_;
  // followed in memory by: cmp_off[B+1], tile_off[B+1]
};

struct PrefillArgs {
  Geometry geo;
  int batch;
  int total_tokens;
  int cmp_rows;  // rows of k_cmp / v_cmp (floor(total / l))
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const float* gates;
  const float* w_k;
  const float* w_v;
  const int* cu;
  void* out;
  uint16_t* k_cmp;
  uint16_t* v_cmp;
  int* sel;
  // workspace views
  int* status;
  Meta* meta;
  int* cmp_off;   // [B+1]
  int* tile_off;  // [B+1]
  float* o_cmp;   // [T, Hq, D]
  float* lse;     // [T, Hq]
  float* scores;  // [T, Hkv, cmp_cap]
  float* sel_scores;  // [T, Hkv, sel_cap] selection-block scores (remap only)
  float* o_win;   // [T, Hq, D] g_win * O_win
  int select_only;  // select-only block attention: routing scores, the own
                    // block forced into the selection, output = selected branch
  int token_select; // token-level top-k (index scores into `scores`, geometry of
                    // the indexer: G = indexer heads, Hkv = 1, D = indexer dim;
                    // `gates` holds the per-token head weights [T, G])
  int split_q;    // PrefillMaps.q_split is valid (Hq >= 16)
  int split_v;    // PrefillMaps.v_split is valid (l' = 64)
};

struct PrefillMaps {
  CUtensorMap q;      // (D, Hq, T) box (64, G, tpt)
  CUtensorMap q_tok;  // (D, Hq, T) box (64, min(16, Hq), 1)
  CUtensorMap q_split;  // (64, Hq, D/64, T) box (64, 16, D/64, 1): [half][head][64]
  CUtensorMap v_split;  // (64, T, D/64, Hkv) box (64, l', D/64, 1): [half][key][64] (l' = 64)
  CUtensorMap kc;     // (D, Hkv, cmp_rows) box (64, 1, 128)
  CUtensorMap vc;
  CUtensorMap k_blk;  // (D, Hkv, T) box (64, 1, l')
  CUtensorMap v_blk;
  CUtensorMap k_win;  // (D, Hkv, T) box (64, 1, 128)
  CUtensorMap v_win;
  CUtensorMap wpl;    // (l D, 2 x 3 x Hkv x D) box (64, 64): the bf16 weight terms
};

struct DecodeArgs {
  Geometry geo;
  int batch;
  int cap;   // cache capacity in tokens (multiple of l and of l')
  int ccap;  // compressed-cache capacity = cap / d
  const uint16_t* q;        // [B, Hq, D]
  const uint16_t* k_cache;  // [B, cap, Hkv, D]
  const uint16_t* v_cache;
  uint16_t* k_cmp;          // [B, ccap, Hkv, D]
  uint16_t* v_cmp;
  const int* seqlens;       // [B]
  const float* gates;       // [B, Hq, 3]
  const float* w_k;
  const float* w_v;
  void* out;                // [B, Hq, D]
  int* sel;                 // [B, Hkv, n] or null
  int* status;
  int select_only;          // select-only block attention: k_cmp is the mean-key cache
                            // [B, cap / l', Hkv, D]; routing scores, the own block
                            // forced in, output = selected branch (no gates)
  // units of the second decode kernel and its workspace records (per
  // (sequence, group) pair: see nsa_decode_b_kernel)
  int ncc_max;              // ceil(ccap / 128): compressed chunks of the longest sequence
  int ncv_max;              // ceil(ncc_max / kUnitChunks): compressed-value units per pair
  int nsl;                  // ceil(selected chunks / kUnitChunks): selected units per pair
  int nwu;                  // ceil(window chunks / kUnitChunks): window units per pair
  int* counters;            // [B * Hkv] finished units per pair (zero at launch)
  int* ws_sel;              // [B * Hkv, n]
  uint8_t* ws_pt;           // [B * Hkv, ncc_max, 4096 B] normalised compressed P^T, bf16
  float* ws_win;            // [B * Hkv, nwu, G * D + 32] window partials
  float* ws_cmp;            // [B * Hkv, ncv_max, G, D]
  float* ws_slc;            // [B * Hkv, nsl, G * D + 32]
};

struct DecodeMaps {
  CUtensorMap q;      // (D, Hq, B) box (64, 16, 1)
  CUtensorMap kc;     // (D, Hkv, ccap, B) box (64, 1, 128, 1)
  CUtensorMap vc;
  CUtensorMap k_blk;  // (D, Hkv, cap, B) box (64, 1, l', 1)
  CUtensorMap v_blk;
  CUtensorMap k_win;  // (D, Hkv, cap, B) box (64, 1, 128, 1)
  CUtensorMap v_win;
};

// Largest number of compressed blocks one decode query may see (all of its
// compressed scores stay in TMEM: 32 chunks of 128 keys x 16 columns).
constexpr int kDecodeMaxCmp = 4096;
// 128-key chunks per unit of the second decode kernel
constexpr int kUnitChunks = 4;

// Complete compressed blocks among the first `len` tokens of a sequence
// (block i covers tokens [i d, i d + l - 1]).
__host__ __device__ __forceinline__ int num_cmp_blocks(int len, int l, int d) {
  return len >= l ? (len - l) / d + 1 : 0;
}

// Selection score of block j (tokens [j l', j l' + l' - 1]) from the group's
// compressed-block scores S(i), i < ncmp: the sum over the visible
// compressed blocks that overlap it, in increasing i.  With l == d == l' it
// is S(j) itself (0 for the incomplete block).
template <typename ScoreFn>
__device__ __forceinline__ float remap_score(const Geometry& g, ScoreFn S, int ncmp, int j) {
  // i d <= (j + 1) l' - 1  and  i d + l - 1 >= j l'
  const int lo_num = j * g.ls - g.l + 1;
  int i0 = lo_num <= 0 ? 0 : (lo_num + g.d - 1) / g.d;
  int i1 = ((j + 1) * g.ls - 1) / g.d;
  if (i1 > ncmp - 1) i1 = ncmp - 1;
  float s = 0.f;
  for (int i = i0; i <= i1; ++i) s += S(i);
  return s;
}

// Sequence of token `tok` (binary search over cu[0..B]).
__device__ __forceinline__ int seq_of_token(const int* cu, int B, int tok) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= tok) lo = mid; else hi = mid - 1;
  }
  return lo;
}
// Index b with off[b] <= x < off[b+1].
__device__ __forceinline__ int seq_of_offset(const int* off, int B, int x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_meta(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_weight_split(const PrefillArgs& a, uint16_t* planes, cudaStream_t s);
cudaError_t launch_compress_tc(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                               cudaStream_t s);
cudaError_t launch_cmp_attn(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                            cudaStream_t s);
cudaError_t launch_topn(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_win(const PrefillArgs& a, const PrefillMaps& m, int num_sms, cudaStream_t s);
cudaError_t launch_slc(const PrefillArgs& a, const PrefillMaps& m, int num_sms, cudaStream_t s);
cudaError_t launch_block_mean(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_block_score(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                               cudaStream_t s);
cudaError_t launch_token_topk(const PrefillArgs& a, int top_k, cudaStream_t s);
cudaError_t launch_token_attn(const PrefillArgs& a, int top_k, cudaStream_t s);
cudaError_t launch_timeout_selftest(int* status, long long cycles, cudaStream_t s);
cudaError_t launch_decode_compress(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_block_mean(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_a(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s);
cudaError_t launch_decode_b(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t s);

}  // namespace nsa
