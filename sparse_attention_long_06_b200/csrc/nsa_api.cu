// Host side of the C ABI declared in include/nsa.h: plan validation,
// workspace layout, TMA descriptor encoding and the launch sequence.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "nsa_internal.cuh"

using namespace nsa;

struct nsa_plan_s {
  nsa_params p;
  Geometry geo;
};

namespace {

thread_local int g_last_launches = 0;

// ---------------------------------------------------------------- profiling hook
constexpr int kMaxProfEvents = 16;
struct Profiler {
  bool enabled = false;
  bool created = false;
  int marks = 0;  // events recorded by the last profiled call
  cudaEvent_t ev[kMaxProfEvents];
};
thread_local Profiler g_prof;

void prof_reset() { g_prof.marks = 0; }
void prof_mark(cudaStream_t s) {
  if (!g_prof.enabled || g_prof.marks >= kMaxProfEvents) return;
  if (!g_prof.created) {
    for (int i = 0; i < kMaxProfEvents; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return;
    g_prof.created = true;
  }
  cudaEventRecord(g_prof.ev[g_prof.marks++], s);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool is_pow2_le16(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

struct PrefillLayout {
  size_t meta, o_cmp, lse, scores, sel_scores, sel, o_win, wplanes, total;
};

// bf16 terms of the compressor weights: [tensor][term][Hkv][D][l D]
size_t weight_plane_bytes(const Geometry& g) {
  return (size_t)2 * 3 * g.Hkv * g.D * (size_t)g.l * g.D * 2;
}

PrefillLayout prefill_layout(const nsa_plan_s* pl) {
  const nsa_params& p = pl->p;
  const Geometry& g = pl->geo;
  const size_t T = (size_t)p.max_total_tokens;
  PrefillLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  take(kHeaderBytes);  // status word at offset 0
  L.meta = take(sizeof(Meta) + 2 * sizeof(int) * ((size_t)p.max_batch + 1));
  L.o_cmp = take(T * g.Hq * g.D * sizeof(float));
  L.lse = take(T * g.Hq * sizeof(float));
  L.scores = take(T * g.Hkv * (size_t)g.cmp_cap * sizeof(float));
  L.sel_scores = take(g.remap ? T * g.Hkv * (size_t)g.sel_cap * sizeof(float) : 0);
  L.sel = take(T * g.Hkv * (size_t)g.n * sizeof(int));
  L.o_win = take(T * g.Hq * g.D * sizeof(float));
  L.wplanes = take(weight_plane_bytes(g));
  L.total = off;
  return L;
}

// Select-only block attention: the plan's geometry with blocks of l' tokens
// as the pooled (routing) blocks; the score table holds max_seqlen / l'
// routing scores per (token, group).
Geometry block_select_geometry(const nsa_plan_s* pl) {
  Geometry g = pl->geo;
  g.l = g.ls;
  g.d = g.ls;
  g.remap = 0;
  g.cmp_cap = pl->p.max_seqlen / g.ls > 0 ? pl->p.max_seqlen / g.ls : 1;
  return g;
}

struct BlockSelectLayout {
  size_t meta, scores, sel, total;
};

BlockSelectLayout block_select_layout(const nsa_plan_s* pl) {
  const nsa_params& p = pl->p;
  const Geometry g = block_select_geometry(pl);
  const size_t T = (size_t)p.max_total_tokens;
  BlockSelectLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  take(kHeaderBytes);
  L.meta = take(sizeof(Meta) + 2 * sizeof(int) * ((size_t)p.max_batch + 1));
  L.scores = take(T * g.Hkv * (size_t)g.cmp_cap * sizeof(float));
  L.sel = take(T * g.Hkv * (size_t)g.n * sizeof(int));
  L.total = off;
  return L;
}

struct DecodeLayout {
  size_t counters, sel, pt, win, cmp, slc, total;
  int ncc_max, ncv_max, nsl, nwu;
};

// Decode workspace for `batch` sequences in a cache of `cap` tokens:
// status header, per-pair unit counters, selection, compressed P^T and the
// fp32 partial records of the second decode kernel.
DecodeLayout decode_layout(const nsa_plan_s* pl, int batch, int cap, bool select_only = false) {
  const Geometry& g = pl->geo;
  DecodeLayout L{};
  const size_t pairs = (size_t)batch * g.Hkv;
  const int ccap = cap / (select_only ? g.ls : g.d);
  L.ncc_max = (ccap + kChunk - 1) / kChunk;
  const int nsc = (g.n + (kChunk >> g.lg_ls) - 1) / (kChunk >> g.lg_ls);
  L.nsl = (nsc + kUnitChunks - 1) / kUnitChunks;
  const int wmax = g.w < cap ? g.w : cap;
  // select-only: selected units only (no compressed values, no window, no P^T)
  L.ncv_max = select_only ? 0 : (L.ncc_max + kUnitChunks - 1) / kUnitChunks;
  L.nwu = select_only ? 0 : ((wmax + kChunk - 1) / kChunk + kUnitChunks - 1) / kUnitChunks;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  take(kHeaderBytes);
  L.counters = take(pairs * sizeof(int));
  L.sel = take(pairs * g.n * sizeof(int));
  L.pt = take(select_only ? 0 : pairs * (size_t)L.ncc_max * 4096);
  L.win = take(pairs * (size_t)L.nwu * (g.G * g.D + 32) * sizeof(float));
  L.cmp = take(pairs * (size_t)L.ncv_max * g.G * g.D * sizeof(float));
  L.slc = take(pairs * (size_t)L.nsl * (g.G * g.D + 32) * sizeof(float));
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- TMA encode
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 3-D bf16 tensor (inner D, middle heads, outer rows), 128-byte swizzled box.
bool encode3d(CUtensorMap* m, const void* base, int D, int heads, long long rows, int box_heads,
              int box_rows) {
  memset(m, 0, sizeof(*m));
  if (rows <= 0) return true;  // never dereferenced
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * heads};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 tensor (D, heads, rows, batch), 128-byte swizzled box (64, 1, box_rows, 1).
bool encode4d(CUtensorMap* m, const void* base, int D, int heads, long long rows, int batch,
              int box_rows) {
  memset(m, 0, sizeof(*m));
  if (rows <= 0 || batch <= 0) return true;
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * heads,
                           (cuuint64_t)D * 2 * heads * rows};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view of a bf16 [rows, heads, D] tensor whose box brings both 64-channel
// halves of `box_rows` consecutive rows of one head (or `box_heads` heads of
// one row) in one copy, laid out [half][row or head][64 channels] in shared
// memory: dims (64 channels, inner, D / 64 halves, outer).  `inner_is_rows`
// picks (rows, heads) or (heads, rows) for the inner/outer dims.  Returns
// false when the driver rejects the map (the kernels then use 3-D boxes).
bool encode_split4d(CUtensorMap* m, const void* base, int D, int heads, long long rows,
                    bool inner_is_rows, int box_inner) {
  memset(m, 0, sizeof(*m));
  if (rows <= 0) return false;
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t row_stride = (cuuint64_t)D * 2 * heads, head_stride = (cuuint64_t)D * 2;
  cuuint64_t dims[4] = {64, inner_is_rows ? (cuuint64_t)rows : (cuuint64_t)heads,
                        (cuuint64_t)(D / 64), inner_is_rows ? (cuuint64_t)heads : (cuuint64_t)rows};
  cuuint64_t strides[3] = {inner_is_rows ? row_stride : head_stride, 128,
                           inner_is_rows ? head_stride : row_stride};
  cuuint32_t box[4] = {64, (cuuint32_t)box_inner, (cuuint32_t)(D / 64), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor (inner `cols`, outer `rows`), 128-byte swizzled box (64, box_rows).
bool encode2d(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows) {
  memset(m, 0, sizeof(*m));
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace

extern "C" {

const char* nsa_strerror(int status) {
  switch (status) {
    case NSA_OK: return "ok";
    case NSA_ERR_INVALID_ARG: return "invalid argument";
    case NSA_ERR_UNSUPPORTED: return "unsupported geometry";
    case NSA_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case NSA_ERR_WORKSPACE: return "workspace missing or too small";
    case NSA_ERR_CUDA: return "CUDA runtime error";
    case NSA_ERR_DEVICE_TIMEOUT: return "device: bounded wait gave up";
    case NSA_ERR_DEVICE_BAD_INPUT: return "device: sequence lengths out of range";
    default: return "unknown status";
  }
}

int nsa_last_launch_count(void) { return g_last_launches; }

int nsa_profile_enable(int enable) {
  g_prof.enabled = enable != 0;
  g_prof.marks = 0;
  return NSA_OK;
}

int nsa_profile_stage_ms(float* ms, int max_stages) {
  if (g_prof.marks < 2) return -1;
  if (cudaEventSynchronize(g_prof.ev[g_prof.marks - 1]) != cudaSuccess) return -1;
  const int n = g_prof.marks - 1;
  for (int i = 0; i < n && i < max_stages && ms; ++i)
    if (cudaEventElapsedTime(&ms[i], g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) return -1;
  return n;
}

int nsa_plan_create(const nsa_params* params, nsa_plan_t* plan_out) {
  if (!params || !plan_out) return NSA_ERR_INVALID_ARG;
  *plan_out = nullptr;
  const nsa_params& p = *params;
  if (p.head_dim <= 0 || p.num_q_heads <= 0 || p.num_kv_heads <= 0 || p.cmp_block <= 0 ||
      p.cmp_stride <= 0 || p.sel_block <= 0 || p.top_n <= 0 || p.window <= 0 ||
      p.max_batch <= 0 || p.max_seqlen <= 0 || p.max_total_tokens < 0 ||
      p.softmax_scale < 0.f || !std::isfinite(p.softmax_scale) ||
      (p.out_dtype != NSA_OUT_BF16 && p.out_dtype != NSA_OUT_F32))
    return NSA_ERR_INVALID_ARG;
  if (p.num_q_heads % p.num_kv_heads != 0) return NSA_ERR_INVALID_ARG;
  if (p.cmp_stride > p.cmp_block || p.cmp_block % p.cmp_stride != 0) return NSA_ERR_INVALID_ARG;
  const int G = p.num_q_heads / p.num_kv_heads;
  if (p.head_dim != 64 && p.head_dim != 128) return NSA_ERR_UNSUPPORTED;
  if (!is_pow2_le16(G)) return NSA_ERR_UNSUPPORTED;
  // compression blocks of 32 or 64 tokens at a stride of 16, 32 or 64 that
  // divides them; selection blocks of 32 or 64 tokens
  if (p.cmp_block != 32 && p.cmp_block != 64) return NSA_ERR_UNSUPPORTED;
  if (p.cmp_stride != 16 && p.cmp_stride != 32 && p.cmp_stride != 64) return NSA_ERR_UNSUPPORTED;
  if (p.sel_block != 32 && p.sel_block != 64) return NSA_ERR_UNSUPPORTED;
  // the selected branch keeps all of one token's selected keys in TMEM (at
  // most 8 chunks of 128 keys) and deals the selection to the 32 lanes of a
  // warp
  if (p.top_n > 8 * (kChunk / p.sel_block) || p.top_n > 32) return NSA_ERR_UNSUPPORTED;
  if (p.max_seqlen < p.cmp_block) return NSA_ERR_INVALID_ARG;
  nsa_plan_s* pl = new (std::nothrow) nsa_plan_s;
  if (!pl) return NSA_ERR_INVALID_ARG;
  pl->p = p;
  Geometry& g = pl->geo;
  g.D = p.head_dim;
  g.Hq = p.num_q_heads;
  g.Hkv = p.num_kv_heads;
  g.G = G;
  g.lg_G = __builtin_ctz(G);
  g.tpt = kTileRows / G;
  g.l = p.cmp_block;
  g.d = p.cmp_stride;
  g.ls = p.sel_block;
  g.lg_ls = __builtin_ctz(p.sel_block);
  g.remap = !(g.d == g.l && g.ls == g.l);
  g.n = p.top_n;
  g.w = p.window;
  g.cmp_cap = num_cmp_blocks(p.max_seqlen, g.l, g.d);
  g.sel_cap = p.max_seqlen / g.ls + 1;
  g.max_seqlen = p.max_seqlen;
  g.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / std::sqrt((float)p.head_dim);
  g.scale_log2 = g.scale * 1.4426950408889634f;
  g.out_f32 = p.out_dtype == NSA_OUT_F32;
  *plan_out = pl;
  return NSA_OK;
}

int nsa_plan(const nsa_params* params, nsa_plan_t* plan_out) {
  return nsa_plan_create(params, plan_out);
}

void nsa_plan_destroy(nsa_plan_t plan) { delete plan; }

size_t nsa_workspace_size(nsa_plan_t plan, int mode) {
  if (!plan) return 0;
  if (mode == NSA_MODE_PREFILL) return prefill_layout(plan).total;
  if (mode == NSA_MODE_DECODE) {
    const int unit = plan->geo.l > plan->geo.ls ? plan->geo.l : plan->geo.ls;
    const int cap = plan->p.max_seqlen / unit * unit;
    return decode_layout(plan, plan->p.max_batch, cap).total;
  }
  if (mode == NSA_MODE_BLOCK_SELECT) return block_select_layout(plan).total;
  if (mode == NSA_MODE_BLOCK_SELECT_DECODE) {
    const int cap = plan->p.max_seqlen / plan->geo.ls * plan->geo.ls;
    return decode_layout(plan, plan->p.max_batch, cap, true).total;
  }
  return 0;
}

int nsa_workspace_region(nsa_plan_t plan, int mode, int region, size_t* offset, size_t* bytes) {
  if (!plan || !offset || !bytes) return NSA_ERR_INVALID_ARG;
  if (mode == NSA_MODE_BLOCK_SELECT) {
    const BlockSelectLayout L = block_select_layout(plan);
    const Geometry g = block_select_geometry(plan);
    const size_t T = (size_t)plan->p.max_total_tokens;
    switch (region) {
      case NSA_WS_STATUS: *offset = 0; *bytes = sizeof(int); break;
      case NSA_WS_SCORES: *offset = L.scores; *bytes = T * g.Hkv * (size_t)g.cmp_cap * sizeof(float); break;
      case NSA_WS_SEL: *offset = L.sel; *bytes = T * g.Hkv * (size_t)g.n * sizeof(int); break;
      default: return NSA_ERR_INVALID_ARG;
    }
    return NSA_OK;
  }
  if (mode != NSA_MODE_PREFILL) return NSA_ERR_INVALID_ARG;
  const PrefillLayout L = prefill_layout(plan);
  const Geometry& g = plan->geo;
  const size_t T = (size_t)plan->p.max_total_tokens;
  switch (region) {
    case NSA_WS_STATUS: *offset = 0; *bytes = sizeof(int); break;
    case NSA_WS_O_CMP: *offset = L.o_cmp; *bytes = T * g.Hq * g.D * sizeof(float); break;
    case NSA_WS_LSE: *offset = L.lse; *bytes = T * g.Hq * sizeof(float); break;
    case NSA_WS_SCORES: *offset = L.scores; *bytes = T * g.Hkv * (size_t)g.cmp_cap * sizeof(float); break;
    case NSA_WS_SEL_SCORES:
      *offset = L.sel_scores;
      *bytes = g.remap ? T * g.Hkv * (size_t)g.sel_cap * sizeof(float) : 0;
      break;
    case NSA_WS_SEL: *offset = L.sel; *bytes = T * g.Hkv * (size_t)g.n * sizeof(int); break;
    case NSA_WS_WIN: *offset = L.o_win; *bytes = T * g.Hq * g.D * sizeof(float); break;
    default: return NSA_ERR_INVALID_ARG;
  }
  return NSA_OK;
}

int nsa_cmp_rows(nsa_plan_t plan, int total_tokens) {
  if (!plan || total_tokens < 0) return -1;
  // sum_b ((T_b - l) / d + 1) <= T_total / d for l >= d
  return total_tokens / plan->geo.d;
}

int nsa_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v, const float* gates,
                const float* w_k, const float* w_v, const int* cu_seqlens, int batch,
                int total_tokens, void* out, void* k_cmp, void* v_cmp, int* sel_idx,
                void* workspace, size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  if (!plan) return NSA_ERR_INVALID_ARG;
  const nsa_params& p = plan->p;
  const Geometry& geo = plan->geo;
  if (batch <= 0 || batch > p.max_batch || total_tokens < 0 ||
      total_tokens > p.max_total_tokens)
    return NSA_ERR_INVALID_ARG;
  if (!cu_seqlens || !workspace) return workspace ? NSA_ERR_INVALID_ARG : NSA_ERR_WORKSPACE;
  const PrefillLayout L = prefill_layout(plan);
  if (workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return NSA_ERR_WORKSPACE;
  const int cmp_rows = total_tokens / geo.d;
  if (total_tokens > 0) {
    if (!q || !k || !v || !gates || !w_k || !w_v || !out) return NSA_ERR_INVALID_ARG;
    if (cmp_rows > 0 && (!k_cmp || !v_cmp)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(w_k) || !aligned16(w_v) || (cmp_rows > 0 && (!aligned16(k_cmp) || !aligned16(v_cmp))) ||
        (reinterpret_cast<uintptr_t>(gates) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(sel_idx) & 3u))
      return NSA_ERR_MISALIGNED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  PrefillArgs a{};
  a.geo = geo;
  a.batch = batch;
  a.total_tokens = total_tokens;
  a.cmp_rows = cmp_rows;
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.gates = gates;
  a.w_k = w_k;
  a.w_v = w_v;
  a.cu = cu_seqlens;
  a.out = out;
  a.k_cmp = static_cast<uint16_t*>(k_cmp);
  a.v_cmp = static_cast<uint16_t*>(v_cmp);
  a.status = reinterpret_cast<int*>(ws);
  a.meta = reinterpret_cast<Meta*>(ws + L.meta);
  a.cmp_off = reinterpret_cast<int*>(ws + L.meta + sizeof(Meta));
  a.tile_off = a.cmp_off + (batch + 1);
  a.o_cmp = reinterpret_cast<float*>(ws + L.o_cmp);
  a.lse = reinterpret_cast<float*>(ws + L.lse);
  a.scores = reinterpret_cast<float*>(ws + L.scores);
  a.sel_scores = reinterpret_cast<float*>(ws + L.sel_scores);
  a.sel = sel_idx ? sel_idx : reinterpret_cast<int*>(ws + L.sel);
  a.o_win = reinterpret_cast<float*>(ws + L.o_win);

  // status word: cleared at the start of every call
  if (cudaMemsetAsync(a.status, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  if (total_tokens == 0) {
    if (cudaMemsetAsync(a.meta, 0, sizeof(Meta), s) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
  }
  PrefillMaps m;
  bool ok = encode3d(&m.q, q, geo.D, geo.Hq, total_tokens, geo.G, geo.tpt) &&
            encode3d(&m.q_tok, q, geo.D, geo.Hq, total_tokens, geo.Hq < 16 ? geo.Hq : 16, 1) &&
            encode3d(&m.kc, k_cmp, geo.D, geo.Hkv, cmp_rows, 1, kChunk) &&
            encode3d(&m.vc, v_cmp, geo.D, geo.Hkv, cmp_rows, 1, kChunk) &&
            encode3d(&m.k_blk, k, geo.D, geo.Hkv, total_tokens, 1, geo.ls) &&
            encode3d(&m.v_blk, v, geo.D, geo.Hkv, total_tokens, 1, geo.ls) &&
            encode3d(&m.k_win, k, geo.D, geo.Hkv, total_tokens, 1, kChunk) &&
            encode3d(&m.v_win, v, geo.D, geo.Hkv, total_tokens, 1, kChunk) &&
            encode2d(&m.wpl, ws + L.wplanes, (long long)geo.l * geo.D, 6LL * geo.Hkv * geo.D, 64);
  if (!ok) return NSA_ERR_CUDA;
  // one-copy query rows (16 heads) and one-copy V blocks (64 keys), when the
  // driver accepts the channel-split maps
  a.split_q = geo.Hq >= 16 && encode_split4d(&m.q_split, q, geo.D, geo.Hq, total_tokens, false, 16);
  a.split_v = geo.ls == 64 && encode_split4d(&m.v_split, v, geo.D, geo.Hkv, total_tokens, true, 64);
  static std::once_flag split_note;
  if ((geo.Hq >= 16 && !a.split_q) || (geo.ls == 64 && !a.split_v))
    std::call_once(split_note, [] {
      fprintf(stderr, "nsa_prefill: channel-split tensor maps rejected by the driver; "
                      "using one copy per 64-channel half\n");
    });
  const int sms = num_sms_current();
  if (sms <= 0) return NSA_ERR_CUDA;

  int launches = 0;
  prof_reset();
  prof_mark(s);
  cudaError_t e = launch_meta(a, s);
  if (e == cudaSuccess) {
    ++launches;
    prof_mark(s);
    e = launch_weight_split(a, reinterpret_cast<uint16_t*>(ws + L.wplanes), s);
  }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_compress_tc(a, m, sms, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_cmp_attn(a, m, sms, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_topn(a, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_win(a, m, sms, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_slc(a, m, sms, s); }
  prof_mark(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "nsa_prefill: launch failed: %s\n", cudaGetErrorString(e));
    return NSA_ERR_CUDA;
  }
  g_last_launches = launches + 1;
  return NSA_OK;
}

namespace {
struct TokenSelectLayout {
  size_t meta, scores, sel, total;
};

// row stride (floats) of the index-score table: rows start on 16 bytes
int token_score_stride(int max_seqlen) { return (max_seqlen + 3) & ~3; }

TokenSelectLayout token_select_layout(const nsa_plan_s* pl, int top_k) {
  const nsa_params& p = pl->p;
  const size_t T = (size_t)p.max_total_tokens;
  TokenSelectLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  take(kHeaderBytes);
  L.meta = take(sizeof(Meta) + 2 * sizeof(int) * ((size_t)p.max_batch + 1));
  L.scores = take(T * (size_t)token_score_stride(p.max_seqlen) * sizeof(float));
  L.sel = take(T * (size_t)top_k * sizeof(int));
  L.total = off;
  return L;
}
}  // namespace

size_t nsa_token_select_workspace_size(nsa_plan_t plan, int top_k) {
  if (!plan || top_k < 1) return 0;
  return token_select_layout(plan, top_k).total;
}

int nsa_token_select_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v,
                             const void* q_index, const float* w_index, const void* k_index,
                             int index_heads, int index_dim, int top_k, const int* cu_seqlens,
                             int batch, int total_tokens, void* out, int* sel_idx,
                             void* workspace, size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  if (!plan) return NSA_ERR_INVALID_ARG;
  const nsa_params& p = plan->p;
  const Geometry& geo = plan->geo;
  if (batch <= 0 || batch > p.max_batch || total_tokens < 0 ||
      total_tokens > p.max_total_tokens || top_k < 1 || top_k > p.max_seqlen || index_heads < 1 ||
      index_dim < 1)
    return NSA_ERR_INVALID_ARG;
  if (!is_pow2_le16(index_heads) || (index_dim != 64 && index_dim != 128) || geo.Hq > 64 ||
      geo.Hkv > (geo.D == 128 ? 4 : 8))
    return NSA_ERR_UNSUPPORTED;
  if (!cu_seqlens || !workspace) return workspace ? NSA_ERR_INVALID_ARG : NSA_ERR_WORKSPACE;
  const TokenSelectLayout L = token_select_layout(plan, top_k);
  if (workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return NSA_ERR_WORKSPACE;
  if (total_tokens > 0) {
    if (!q || !k || !v || !q_index || !w_index || !k_index || !out) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_index) ||
        !aligned16(k_index) || !aligned16(out) || (reinterpret_cast<uintptr_t>(w_index) & 3u) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(sel_idx) & 3u))
      return NSA_ERR_MISALIGNED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the indexer's geometry: its heads are the columns of a token, one key head
  Geometry gi = geo;
  gi.D = index_dim;
  gi.Hq = index_heads;
  gi.Hkv = 1;
  gi.G = index_heads;
  gi.lg_G = __builtin_ctz(index_heads);
  gi.tpt = kTileRows / index_heads;
  gi.l = gi.d = gi.ls = 1;
  gi.lg_ls = 0;
  gi.remap = 0;
  gi.cmp_cap = token_score_stride(p.max_seqlen);  // row stride of the index-score table
  PrefillArgs ai{};
  ai.geo = gi;
  ai.batch = batch;
  ai.total_tokens = total_tokens;
  ai.cmp_rows = total_tokens;
  ai.q = static_cast<const uint16_t*>(q_index);
  ai.k_cmp = static_cast<uint16_t*>(const_cast<void*>(k_index));
  ai.gates = w_index;
  ai.cu = cu_seqlens;
  ai.status = reinterpret_cast<int*>(ws);
  ai.meta = reinterpret_cast<Meta*>(ws + L.meta);
  ai.cmp_off = reinterpret_cast<int*>(ws + L.meta + sizeof(Meta));
  ai.tile_off = ai.cmp_off + (batch + 1);
  ai.scores = reinterpret_cast<float*>(ws + L.scores);
  ai.sel = sel_idx ? sel_idx : reinterpret_cast<int*>(ws + L.sel);
  ai.token_select = 1;
  PrefillArgs am = ai;  // the main attention: the plan's geometry
  am.geo = geo;
  am.q = static_cast<const uint16_t*>(q);
  am.k = static_cast<const uint16_t*>(k);
  am.v = static_cast<const uint16_t*>(v);
  am.out = out;
  am.token_select = 0;

  if (cudaMemsetAsync(ai.status, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  if (total_tokens == 0) {
    if (cudaMemsetAsync(ai.meta, 0, sizeof(Meta), s) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
  }
  PrefillMaps m;
  memset(&m, 0, sizeof(m));
  bool ok = encode3d(&m.q, q_index, index_dim, index_heads, total_tokens, index_heads, gi.tpt) &&
            encode3d(&m.kc, k_index, index_dim, 1, total_tokens, 1, kChunk);
  if (!ok) return NSA_ERR_CUDA;
  const int sms = num_sms_current();
  if (sms <= 0) return NSA_ERR_CUDA;
  int launches = 0;
  prof_reset();
  prof_mark(s);
  cudaError_t e = launch_meta(ai, s);
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_block_score(ai, m, sms, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_token_topk(ai, top_k, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_token_attn(am, top_k, s); }
  prof_mark(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "nsa_token_select_prefill: launch failed: %s\n", cudaGetErrorString(e));
    return NSA_ERR_CUDA;
  }
  g_last_launches = launches + 1;
  return NSA_OK;
}

int nsa_block_rows(nsa_plan_t plan, int total_tokens) {
  if (!plan || total_tokens < 0) return -1;
  return total_tokens / plan->geo.ls;
}

int nsa_block_select_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v,
                             const int* cu_seqlens, int batch, int total_tokens, void* out,
                             void* k_mean, int* sel_idx, void* workspace, size_t workspace_bytes,
                             void* stream) {
  g_last_launches = 0;
  if (!plan) return NSA_ERR_INVALID_ARG;
  const nsa_params& p = plan->p;
  const Geometry geo = block_select_geometry(plan);
  if (batch <= 0 || batch > p.max_batch || total_tokens < 0 ||
      total_tokens > p.max_total_tokens)
    return NSA_ERR_INVALID_ARG;
  if (!cu_seqlens || !workspace) return workspace ? NSA_ERR_INVALID_ARG : NSA_ERR_WORKSPACE;
  const BlockSelectLayout L = block_select_layout(plan);
  if (workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return NSA_ERR_WORKSPACE;
  const int rows = total_tokens / geo.ls;
  if (total_tokens > 0) {
    if (!q || !k || !v || !out) return NSA_ERR_INVALID_ARG;
    if (rows > 0 && !k_mean) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (rows > 0 && !aligned16(k_mean)) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) ||
        (reinterpret_cast<uintptr_t>(sel_idx) & 3u))
      return NSA_ERR_MISALIGNED;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  PrefillArgs a{};
  a.geo = geo;
  a.batch = batch;
  a.total_tokens = total_tokens;
  a.cmp_rows = rows;
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.cu = cu_seqlens;
  a.out = out;
  a.k_cmp = static_cast<uint16_t*>(k_mean);
  a.status = reinterpret_cast<int*>(ws);
  a.meta = reinterpret_cast<Meta*>(ws + L.meta);
  a.cmp_off = reinterpret_cast<int*>(ws + L.meta + sizeof(Meta));
  a.tile_off = a.cmp_off + (batch + 1);
  a.scores = reinterpret_cast<float*>(ws + L.scores);
  a.sel = sel_idx ? sel_idx : reinterpret_cast<int*>(ws + L.sel);
  a.select_only = 1;

  if (cudaMemsetAsync(a.status, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  if (total_tokens == 0) {
    if (cudaMemsetAsync(a.meta, 0, sizeof(Meta), s) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
  }
  PrefillMaps m;
  memset(&m, 0, sizeof(m));
  bool ok = encode3d(&m.q, q, geo.D, geo.Hq, total_tokens, geo.G, geo.tpt) &&
            encode3d(&m.q_tok, q, geo.D, geo.Hq, total_tokens, geo.Hq < 16 ? geo.Hq : 16, 1) &&
            encode3d(&m.kc, k_mean, geo.D, geo.Hkv, rows, 1, kChunk) &&
            encode3d(&m.k_blk, k, geo.D, geo.Hkv, total_tokens, 1, geo.ls) &&
            encode3d(&m.v_blk, v, geo.D, geo.Hkv, total_tokens, 1, geo.ls);
  if (!ok) return NSA_ERR_CUDA;
  a.split_q = geo.Hq >= 16 && encode_split4d(&m.q_split, q, geo.D, geo.Hq, total_tokens, false, 16);
  a.split_v = geo.ls == 64 && encode_split4d(&m.v_split, v, geo.D, geo.Hkv, total_tokens, true, 64);
  const int sms = num_sms_current();
  if (sms <= 0) return NSA_ERR_CUDA;

  int launches = 0;
  prof_reset();
  prof_mark(s);
  cudaError_t e = launch_meta(a, s);
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_block_mean(a, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_block_score(a, m, sms, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_topn(a, s); }
  if (e == cudaSuccess) { ++launches; prof_mark(s); e = launch_slc(a, m, sms, s); }
  prof_mark(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "nsa_block_select_prefill: launch failed: %s\n", cudaGetErrorString(e));
    return NSA_ERR_CUDA;
  }
  g_last_launches = launches + 1;
  return NSA_OK;
}

int nsa_decode(nsa_plan_t plan, const void* q, const void* k_cache, const void* v_cache,
               void* k_cmp_cache, void* v_cmp_cache, const int* seqlens, int batch,
               int cache_capacity, const float* gates, const float* w_k, const float* w_v,
               void* out, int* sel_idx, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  if (!plan) return NSA_ERR_INVALID_ARG;
  const nsa_params& p = plan->p;
  const Geometry& geo = plan->geo;
  if (batch <= 0 || batch > p.max_batch || cache_capacity <= 0 ||
      cache_capacity > p.max_seqlen || cache_capacity % geo.l != 0 ||
      cache_capacity % geo.ls != 0)
    return NSA_ERR_INVALID_ARG;
  // all of one query's compressed scores and window keys stay in TMEM: at
  // most 4096 compressed blocks, 8 window chunks of 128 keys
  if (num_cmp_blocks(cache_capacity, geo.l, geo.d) > kDecodeMaxCmp || geo.w > 8 * kChunk)
    return NSA_ERR_UNSUPPORTED;
  if (!workspace) return NSA_ERR_WORKSPACE;
  const DecodeLayout DL = decode_layout(plan, batch, cache_capacity);
  if (workspace_bytes < DL.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return NSA_ERR_WORKSPACE;
  if (!q || !k_cache || !v_cache || !k_cmp_cache || !v_cmp_cache || !seqlens || !gates || !w_k ||
      !w_v || !out)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_cmp_cache) ||
      !aligned16(v_cmp_cache) || !aligned16(w_k) || !aligned16(w_v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(gates) & 3u) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u))
    return NSA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.geo = geo;
  a.batch = batch;
  a.cap = cache_capacity;
  a.ccap = cache_capacity / geo.d;
  a.q = static_cast<const uint16_t*>(q);
  a.k_cache = static_cast<const uint16_t*>(k_cache);
  a.v_cache = static_cast<const uint16_t*>(v_cache);
  a.k_cmp = static_cast<uint16_t*>(k_cmp_cache);
  a.v_cmp = static_cast<uint16_t*>(v_cmp_cache);
  a.seqlens = seqlens;
  a.gates = gates;
  a.w_k = w_k;
  a.w_v = w_v;
  a.out = out;
  a.sel = sel_idx;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  a.ncc_max = DL.ncc_max;
  a.ncv_max = DL.ncv_max;
  a.nsl = DL.nsl;
  a.nwu = DL.nwu;
  a.counters = reinterpret_cast<int*>(ws + DL.counters);
  a.ws_sel = reinterpret_cast<int*>(ws + DL.sel);
  a.ws_pt = ws + DL.pt;
  a.ws_win = reinterpret_cast<float*>(ws + DL.win);
  a.ws_cmp = reinterpret_cast<float*>(ws + DL.cmp);
  a.ws_slc = reinterpret_cast<float*>(ws + DL.slc);
  DecodeMaps m;
  bool ok = encode3d(&m.q, q, geo.D, geo.Hq, batch, geo.Hq < 16 ? geo.Hq : 16, 1) &&
            encode4d(&m.kc, k_cmp_cache, geo.D, geo.Hkv, a.ccap, batch, kChunk) &&
            encode4d(&m.vc, v_cmp_cache, geo.D, geo.Hkv, a.ccap, batch, kChunk) &&
            encode4d(&m.k_blk, k_cache, geo.D, geo.Hkv, cache_capacity, batch, geo.ls) &&
            encode4d(&m.v_blk, v_cache, geo.D, geo.Hkv, cache_capacity, batch, geo.ls) &&
            encode4d(&m.k_win, k_cache, geo.D, geo.Hkv, cache_capacity, batch, kChunk) &&
            encode4d(&m.v_win, v_cache, geo.D, geo.Hkv, cache_capacity, batch, kChunk);
  if (!ok) return NSA_ERR_CUDA;
  // status word and per-pair unit counters start at zero
  if (cudaMemsetAsync(ws, 0, DL.counters + (size_t)batch * geo.Hkv * sizeof(int), s) != cudaSuccess)
    return NSA_ERR_CUDA;
  prof_reset();
  prof_mark(s);
  cudaError_t e = launch_decode_compress(a, s);
  if (e == cudaSuccess) {
    prof_mark(s);
    e = launch_decode_a(a, m, s);
  }
  if (e == cudaSuccess) {
    prof_mark(s);
    e = launch_decode_b(a, m, s);
  }
  prof_mark(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "nsa_decode: launch failed: %s\n", cudaGetErrorString(e));
    return NSA_ERR_CUDA;
  }
  g_last_launches = 3;
  return NSA_OK;
}

int nsa_block_select_decode(nsa_plan_t plan, const void* q, const void* k_cache,
                            const void* v_cache, void* k_mean_cache, const int* seqlens, int batch,
                            int cache_capacity, void* out, int* sel_idx, void* workspace,
                            size_t workspace_bytes, void* stream) {
  g_last_launches = 0;
  if (!plan) return NSA_ERR_INVALID_ARG;
  const nsa_params& p = plan->p;
  const Geometry& geo = plan->geo;
  if (batch <= 0 || batch > p.max_batch || cache_capacity <= 0 ||
      cache_capacity > p.max_seqlen || cache_capacity % geo.ls != 0)
    return NSA_ERR_INVALID_ARG;
  // all of one query's routing scores stay on chip: at most 4096 blocks
  if (cache_capacity / geo.ls > kDecodeMaxCmp) return NSA_ERR_UNSUPPORTED;
  if (!workspace) return NSA_ERR_WORKSPACE;
  const DecodeLayout DL = decode_layout(plan, batch, cache_capacity, true);
  if (workspace_bytes < DL.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return NSA_ERR_WORKSPACE;
  if (!q || !k_cache || !v_cache || !k_mean_cache || !seqlens || !out) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_mean_cache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel_idx) & 3u))
    return NSA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.geo = geo;
  a.batch = batch;
  a.cap = cache_capacity;
  a.ccap = cache_capacity / geo.ls;
  a.q = static_cast<const uint16_t*>(q);
  a.k_cache = static_cast<const uint16_t*>(k_cache);
  a.v_cache = static_cast<const uint16_t*>(v_cache);
  a.k_cmp = static_cast<uint16_t*>(k_mean_cache);
  a.seqlens = seqlens;
  a.out = out;
  a.sel = sel_idx;
  a.select_only = 1;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  a.ncc_max = DL.ncc_max;
  a.ncv_max = DL.ncv_max;
  a.nsl = DL.nsl;
  a.nwu = DL.nwu;
  a.counters = reinterpret_cast<int*>(ws + DL.counters);
  a.ws_sel = reinterpret_cast<int*>(ws + DL.sel);
  a.ws_pt = ws + DL.pt;
  a.ws_win = reinterpret_cast<float*>(ws + DL.win);
  a.ws_cmp = reinterpret_cast<float*>(ws + DL.cmp);
  a.ws_slc = reinterpret_cast<float*>(ws + DL.slc);
  DecodeMaps m;
  memset(&m, 0, sizeof(m));
  bool ok = encode3d(&m.q, q, geo.D, geo.Hq, batch, geo.Hq < 16 ? geo.Hq : 16, 1) &&
            encode4d(&m.kc, k_mean_cache, geo.D, geo.Hkv, a.ccap, batch, kChunk) &&
            encode4d(&m.k_blk, k_cache, geo.D, geo.Hkv, cache_capacity, batch, geo.ls) &&
            encode4d(&m.v_blk, v_cache, geo.D, geo.Hkv, cache_capacity, batch, geo.ls);
  if (!ok) return NSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, DL.counters + (size_t)batch * geo.Hkv * sizeof(int), s) != cudaSuccess)
    return NSA_ERR_CUDA;
  prof_reset();
  prof_mark(s);
  cudaError_t e = launch_decode_block_mean(a, s);
  if (e == cudaSuccess) {
    prof_mark(s);
    e = launch_decode_a(a, m, s);
  }
  if (e == cudaSuccess) {
    prof_mark(s);
    e = launch_decode_b(a, m, s);
  }
  prof_mark(s);
  if (e != cudaSuccess) {
    fprintf(stderr, "nsa_block_select_decode: launch failed: %s\n", cudaGetErrorString(e));
    return NSA_ERR_CUDA;
  }
  g_last_launches = 3;
  return NSA_OK;
}

int nsa_read_device_status(const void* workspace, void* stream) {
  if (!workspace) return NSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return NSA_ERR_CUDA;
  int st = 0;
  if (cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return NSA_ERR_CUDA;
  if (cudaMemset(const_cast<void*>(workspace), 0, sizeof(int)) != cudaSuccess) return NSA_ERR_CUDA;
  return st;
}

int nsa_selftest_timeout(void* workspace, size_t workspace_bytes, long long cycles,
                         void* stream) {
  if (!workspace || workspace_bytes < sizeof(int)) return NSA_ERR_WORKSPACE;
  if (cycles <= 0 || cycles > (1LL << 34)) return NSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  if (launch_timeout_selftest(status, cycles, s) != cudaSuccess) return NSA_ERR_CUDA;
  return NSA_OK;
}

}  // extern "C"
