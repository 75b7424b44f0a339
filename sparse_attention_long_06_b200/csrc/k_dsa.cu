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
// Each query token t selects the top_k of its t + 1 index scores (score
// descending, ties to the lower token), written in ascending token order and
// padded with -1 when t + 1 < top_k.
//
// Short rows (at most 1024 candidates, top_k <= 32): one warp per row, the
// register path of the block selection (its 8-bit radix select when more
// keys than the register path ranks reach its bound).
__global__ void __launch_bounds__(256) nsa_token_topk_short_kernel(PrefillArgs a, int top_k) {
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
  if (warp_topn_regs(score, ncand, ncand, top_k, cand_all[warp], put)) return;
  warp_topn(score, ncand, ncand, top_k, hist_all[warp], put);
}

// Rows of any length: one CTA per row, rows taken from the last token back
// so that the longest rows of a sequence start first.  The row (16-byte
// aligned: the table's row stride is a multiple of four) is read as float4.
// A radix select on the 32-bit order-preserving score key with digits of
// 11, 11 and 10 bits finds the key of the top_k-th largest score: each pass
// histograms, in shared memory, the digit of the keys that share the prefix
// found so far (one shared atomic per key: the hardware serialises lanes
// that hit the same bin, which measured faster than aggregating them with
// match.any first), and a block scan over the bins picks the digit holding
// the remaining rank.  The passes stop early once every key of that digit is
// taken.  A last pass compacts the row in token order: a key above the
// threshold is taken, a key equal to it while fewer than the remaining rank
// of equal keys have been taken before it; one block scan per tile gives
// each taken token its output position.
namespace {

constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkBins = 2048;
constexpr int kTkBinsPerThread = kTkBins / kTkThreads;

// Exclusive prefix of v over the CTA's threads in thread order; `total`
// receives the sum over all threads.
__device__ __forceinline__ unsigned tk_excl_scan(unsigned v, unsigned* wsum, unsigned& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  unsigned before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kTkWarps; ++w) {
    const unsigned x = wsum[w];
    before += w < warp ? x : 0u;
    tot += x;
  }
  __syncthreads();
  total = tot;
  return before + inc - v;
}

__device__ __forceinline__ float4 tk_load(const float* S, int q, int nq) {
  return q < nq ? __ldg(reinterpret_cast<const float4*>(S) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// The order-preserving key of score_key in fewer operations: the sign bit
// spread over the word flips every bit of a negative score and only the top
// bit of a non-negative one; -0 takes the key of +0.
__device__ __forceinline__ uint32_t tk_key(float s) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t k = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
  return b == 0x80000000u ? 0x80000000u : k;
}

// One histogram pass of the radix select over the row's candidates: the
// digit (x >> SHIFT) & DMASK of every key x that shares `prefix` (under
// `pmask`; the first pass has no prefix).  `vmask(q)` gives the candidate
// scores of float4 word q (bits 0..3).
template <int SHIFT, uint32_t DMASK, bool FIRST, typename VMask>
__device__ __forceinline__ void tk_hist_pass(const float* S, int nq, VMask vmask, uint32_t prefix,
                                             uint32_t pmask, unsigned* hist) {
  const int tid = threadIdx.x;
  for (int base = 0; base < nq; base += 4 * kTkThreads) {
    float4 v[4];
    uint32_t vm[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = base + u * kTkThreads + tid;
      v[u] = tk_load(S, q, nq);
      vm[u] = vmask(q);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = tk_key(f[e]);
        const bool in = ((vm[u] >> e) & 1u) && (FIRST || (x & pmask) == prefix);
        if (in) atomicAdd(&hist[(x >> SHIFT) & DMASK], 1u);
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kTkThreads) nsa_token_topk_kernel(PrefillArgs a, int top_k) {
  if (a.meta->bad) return;
  __shared__ unsigned hist[kTkBins];
  __shared__ unsigned wsum[kTkWarps];
  __shared__ unsigned ctl[2];
  const int tid = threadIdx.x;
  const int tg = a.total_tokens - 1 - (int)blockIdx.x;
  const int b = seq_of_token(a.cu, a.batch, tg);
  const int ncand = tg - __ldg(a.cu + b) + 1;
  const float* S = a.scores + (size_t)tg * a.geo.cmp_cap;
  int* out = a.sel + (size_t)tg * top_k;
  if (ncand <= top_k) {
    for (int j = tid; j < top_k; j += kTkThreads) out[j] = j < ncand ? j : -1;
    return;
  }
  const int nq = (ncand + 3) >> 2;  // float4 words of the row
  // candidate scores of word q: all four below ncand / 4, the low ncand % 4
  // of the word holding the row's end, none past it
  const int nfull = ncand >> 2;
  const uint32_t tail = (1u << (ncand & 3)) - 1u;
  auto vmask = [=](int q) -> uint32_t { return q < nfull ? 0xFu : (q == nfull ? tail : 0u); };
  uint32_t prefix = 0, pmask = 0;
  unsigned k = (unsigned)top_k;  // rank still to be found inside the prefix class
  int shift = 21;
  for (int pass = 0; pass < 3; ++pass) {
    shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 1023u : 2047u;
    for (int i = tid; i < kTkBins; i += kTkThreads) hist[i] = 0;
    __syncthreads();
    if (pass == 0) tk_hist_pass<21, 2047u, true>(S, nq, vmask, prefix, pmask, hist);
    else if (pass == 1) tk_hist_pass<10, 2047u, false>(S, nq, vmask, prefix, pmask, hist);
    else tk_hist_pass<0, 1023u, false>(S, nq, vmask, prefix, pmask, hist);
    __syncthreads();
    // thread i owns bins [i * 4, i * 4 + 4); higher threads hold higher digits
    unsigned c[kTkBinsPerThread], mine = 0;
#pragma unroll
    for (int e = 0; e < kTkBinsPerThread; ++e) {
      c[e] = hist[tid * kTkBinsPerThread + e];
      mine += c[e];
    }
    unsigned total;
    const unsigned excl = tk_excl_scan(mine, wsum, total);
    const unsigned above = total - excl - mine;  // keys in the class with a higher digit
    if (above < k && k <= above + mine) {
      unsigned acc = above;
      int d = tid * kTkBinsPerThread;
#pragma unroll
      for (int e = kTkBinsPerThread - 1; e >= 0; --e) {
        if (acc + c[e] >= k) {
          d = tid * kTkBinsPerThread + e;
          break;
        }
        acc += c[e];
      }
      ctl[0] = (unsigned)d;
      ctl[1] = acc;
    }
    __syncthreads();
    const uint32_t digit = ctl[0];
    k -= ctl[1];
    prefix |= digit << shift;
    pmask |= dmask << shift;
    const bool all_taken = hist[digit] == k;
    __syncthreads();
    if (all_taken) break;
  }
  // keys compared on their bits from `shift` up: above thr taken, the first
  // `krem` equal to it taken
  const uint32_t thr = prefix >> shift;
  const unsigned krem = k;
  unsigned written = 0, ties = 0;
  float4 nxt = tk_load(S, tid, nq);
  for (int base = 0; base < nq && written < (unsigned)top_k; base += kTkThreads) {
    const float4 cur = nxt;
    nxt = tk_load(S, base + kTkThreads + tid, nq);
    const int j0 = 4 * (base + tid);
    const float f[4] = {cur.x, cur.y, cur.z, cur.w};
    const uint32_t vm = vmask(base + tid);
    unsigned gtm = 0, eqm = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t xt = tk_key(f[e]) >> shift;
      const bool valid = (vm >> e) & 1u;
      gtm |= (valid && xt > thr) ? 1u << e : 0u;
      eqm |= (valid && xt == thr) ? 1u << e : 0u;
    }
    unsigned tot;
    const unsigned excl = tk_excl_scan(((unsigned)__popc(eqm) << 16) | (unsigned)__popc(gtm), wsum, tot);
    const unsigned rem = krem > ties ? krem - ties : 0u;  // equal keys still to take
    unsigned eqb = excl >> 16;
    unsigned pos = written + (excl & 0xFFFFu) + min(eqb, rem);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      bool take = (gtm >> e) & 1u;
      if ((eqm >> e) & 1u) take = eqb++ < rem;
      if (take) {
        if (pos < (unsigned)top_k) out[pos] = j0 + e;
        ++pos;
      }
    }
    written += (tot & 0xFFFFu) + min(tot >> 16, rem);
    ties += tot >> 16;
  }
  for (unsigned j = written + tid; j < (unsigned)top_k; j += kTkThreads) out[j] = -1;
}

// ------------------------------------------------------------------ attention
// One CTA per query token, one warp per KV group: the group's G <= 16 heads
// are the 16 rows of mma.sync m16n8k16 bf16 products with fp32 accumulators
// (rows past G are zero queries whose results are dropped).  The selected
// tokens are taken 32 at a time; their keys and values for every group are
// copied (16-byte cp.async, a ring of three steps: two in flight while one is
// computed; each step's positions are loaded one step before its copies are
// issued) into shared memory rows padded to D + 8 elements, so that the
// eight rows an operand fragment spans fall in different banks.  Per step
// and warp: S = Q K^T (queries as A fragments kept in registers, keys read
// as B fragments), an online softmax on the accumulator fragments (row
// statistics over the four threads of a quad), then O += P V with P
// re-packed from the S fragments as A fragments and V read by
// ldmatrix.trans.  The chosen rows are single 256-byte rows at random
// positions; 16-byte cp.async moved them faster than bulk copies or TMA
// row gathers (tile::gather4).
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
struct TokenAttnCfg {
  static constexpr int RS = D + 8;                          // padded row, elements
  static constexpr int kThreads = HKV * 32;
  static constexpr int kRows = HKV * kDsaKeys;              // rows of one step
  static constexpr int kBufBytes = kRows * RS * 2;          // keys (or values) of one step
  static constexpr int kStages = 3;                         // ring depth
  static constexpr int kSmem = 2 * kStages * kBufBytes;
  static constexpr int CPR = D / 8;                         // 16-byte chunks of a row
  static constexpr int RPI = kThreads / CPR;                // rows copied per pass
  static constexpr int JK = kDsaKeys / RPI;                 // distinct keys per thread
  static_assert(kThreads % CPR == 0 && kDsaKeys % RPI == 0, "copy mapping");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int D, int HKV>
__global__ void __launch_bounds__(HKV * 32) nsa_token_attn_kernel(PrefillArgs a, int top_k) {
  if (a.meta->bad) return;
  using C = TokenAttnCfg<D, HKV>;
  constexpr int RS = C::RS, NST = C::kStages, kBufBytes = C::kBufBytes;
  constexpr int KS = D / 16;                        // k-steps of q . k
  constexpr int NT = D / 8;                         // n-tiles of O
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* kbuf = sm;                               // [NST][HKV][keys][RS]
  uint8_t* vbuf = sm + NST * kBufBytes;             // [NST][HKV][keys][RS]
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
  // thread i copies chunk i % CPR of rows i / CPR + RPI * j: keys
  // i / CPR + RPI * jk of every group
  const int c8 = threadIdx.x % C::CPR, r0 = threadIdx.x / C::CPR;
  // the selected positions of a step, loaded one step before its copies
  // are issued so that the load's latency is hidden behind a step's math
  auto load_sel = [&](int step, int (&sv)[C::JK]) {
#pragma unroll
    for (int jk = 0; jk < C::JK; ++jk) {
      const int i = step * kDsaKeys + r0 + C::RPI * jk;
      sv[jk] = i < nsel ? __ldg(sel + i) : -1;
    }
  };
  auto issue = [&](int step, const int (&sv)[C::JK]) {
    if (step < nsteps) {
      const int buf = step % NST;
      const uint32_t kb = smem_u32(kbuf + buf * kBufBytes), vb = smem_u32(vbuf + buf * kBufBytes);
#pragma unroll
      for (int gg = 0; gg < HKV; ++gg) {
#pragma unroll
        for (int jk = 0; jk < C::JK; ++jk) {
          const int row = gg * kDsaKeys + r0 + C::RPI * jk;
          const bool ok = sv[jk] >= 0;
          const size_t src = ((size_t)(cu0 + (ok ? sv[jk] : 0)) * HKV + gg) * D + c8 * 8;
          cp_async16(kb + (row * RS + c8 * 8) * 2, a.k + src, ok);
          cp_async16(vb + (row * RS + c8 * 8) * 2, a.v + src, ok);
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");  // empty past the last step
  };

  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[n][c] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows gid, gid + 8
  const float sl2 = a.geo.scale_log2;
  int sv[C::JK];
#pragma unroll
  for (int st = 0; st < NST - 1; ++st) {
    load_sel(st, sv);
    issue(st, sv);
  }
  load_sel(NST - 1, sv);
  for (int step = 0; step < nsteps; ++step) {
    const int buf = step % NST;
    // one group committed per step: the NST - 2 after this step's may pend
    asm volatile("cp.async.wait_group %0;" ::"n"(NST - 2) : "memory");
    __syncthreads();  // this step's rows visible; step - 1's buffer free
    issue(step + NST - 1, sv);
    load_sel(step + NST, sv);
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
        const bool on = step * kDsaKeys + key < nsel;
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
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
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
  const size_t smem = TokenAttnCfg<D, HKV>::kSmem;
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
  if (a.geo.cmp_cap <= 1024 && top_k <= 32)
    nsa_token_topk_short_kernel<<<(unsigned)((a.total_tokens + 7) / 8), 256, 0, s>>>(a, top_k);
  else
    nsa_token_topk_kernel<<<(unsigned)a.total_tokens, kTkThreads, 0, s>>>(a, top_k);
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
      default: return launch_token_attn_t<128, 4>(a, top_k, s);  // Hkv <= 4 at D = 128
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
