// Selected-block attention (step 5) and the gate-combine epilogue (step 7).
//
//   step 5 ("DeepSeek NSA config.toml" page, section 3, select_block_size and
//   select_top_k; "DeepSeek NSA in manufacturing" page, section on what
//   dynamic sparsity sparsifies: token-level attention inside the selected
//   blocks): per query head, softmax over the tokens u <= t of the n blocks
//   chosen for the head's KV group, O_slc = sum p v;
//   step 7 (config page, sections 1 and 3, learned gate aggregation):
//   out = g_cmp O_cmp + g_slc O_slc + g_win O_win, where O_cmp comes from the
//   compressed-branch kernel and g_win O_win from the window kernel.
//
// One job = one (token, KV group): its G query heads share the n selected
// blocks, which are loaded once by TMA.  The heads are too few for an M >= 64
// operand, so both products are swapped: S^T = K_blk Q_t^T (M = 128 keys on
// TMEM lanes, N = 16 head columns) and O^T += V_blk^T P^T (M = D channels on
// TMEM lanes).  A persistent CTA per SM takes every gridDim-th job of the
// group-major job list (all tokens of group 0 first, so that one group's K/V
// stays hot in L2).
// Warp roles (384 threads):
//   0  K producer: the token's 16 query rows and the K halves (128 keys x 64
//      channels per ring slot) of its selected blocks;
//   1  QK issuer: S^T into the TMEM score buffer of the job's warpgroup;
//   2  V producer: 64 keys x D channels per ring slot;
//   3  PV issuer: O^T into one of four 16-column TMEM output slots;
//   4..7, 8..11  two softmax warpgroups taking alternate jobs: a two-sweep
//      softmax over the job's keys (per-head maximum, then exp2, sums and P^T
//      in shared memory), then, one job later, the output epilogue of their
//      previous job (thread = channel).
// K and V move through separate rings and separate issuers, so the QK^T of
// the next jobs overlaps the PV of the current one, and the softmax of one
// warpgroup overlaps the epilogue of the other.
#include <cuda_bf16.h>

#include "nsa_internal.cuh"
#include "sm100.cuh"
#include "softmax_util.cuh"

namespace nsa {
using namespace sm100;

namespace {

template <int D>
struct SlcLayout {
  static constexpr int kQSlots = 2;
  static constexpr int kQBytes = 16 * D * 2;  // 16 query rows
  static constexpr int kKSlots = 4;
  static constexpr int kKBytes = kChunk * 64 * 2;  // 128 keys x 64 channels
  static constexpr int kVSlots = D == 128 ? 5 : 8;
  static constexpr int kVBytes = 64 * D * 2;  // 64 keys x D channels
  static constexpr int kPBytes = 8 * 4096;    // P^T: up to 8 chunks x 128 keys x 16 heads
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQSlots * kQBytes;
  static constexpr int kV = kK + kKSlots * kKBytes;
  static constexpr int kP = kV + kVSlots * kVBytes;  // 2 buffers (one per warpgroup)
  static constexpr int kRed = kP + 2 * kPBytes;      // float [2 warpgroups][2][64]
  static constexpr int kInv = kRed + 2 * 2 * 64 * 4; // float [4 output slots][16]
  static constexpr int kBars = kInv + 4 * 16 * 4;
  static constexpr int kEnd = kBars + 64 * 8;
  static constexpr int kSmem = kEnd;
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kP % 1024 == 0, "swizzle alignment");
  static_assert(kSmem <= 232448, "shared memory budget");
  // the PV operand V^T is 128 channels (two 64-channel halves kVBytes / 2
  // apart); with D = 64 its second half reads past the slot, still inside
  // shared memory
  static_assert(kV + kVSlots * kVBytes + (D == 64 ? kVBytes : 0) <= kEnd, "PV operand inside smem");
};

constexpr int kSlcThreads = 384;
constexpr uint32_t kColO = 256;  // four 16-column output slots

struct SlcJob {
  int valid, row, g, t, cu0;
};

// Job J of the group-major list: token row J % T_total of group J / T_total.
__device__ __forceinline__ SlcJob slc_job(const PrefillArgs& a, long long J) {
  SlcJob j{};
  const long long total = a.total_tokens;
  if (J >= total * a.geo.Hkv) return j;
  j.valid = 1;
  j.g = static_cast<int>(J / total);
  j.row = static_cast<int>(J - j.g * total);
  const int b = seq_of_token(a.cu, a.batch, j.row);
  j.cu0 = __ldg(a.cu + b);
  j.t = j.row - j.cu0;
  return j;
}

__device__ __forceinline__ int slc_jobs_of_cta(const PrefillArgs& a) {
  const long long total = (long long)a.total_tokens * a.geo.Hkv;
  if (blockIdx.x >= total) return 0;
  return static_cast<int>((total - 1 - blockIdx.x) / gridDim.x + 1);
}

// Selection entry `lane` of job j (or -1), read by every lane of a warp.
__device__ __forceinline__ int job_sel(const PrefillArgs& a, const SlcJob& j, int lane) {
  if (!j.valid || lane >= a.geo.n) return -1;
  return __ldg(a.sel + ((size_t)j.row * a.geo.Hkv + j.g) * a.geo.n + lane);
}

template <int D>
__global__ void __launch_bounds__(kSlcThreads, 1)
    nsa_slc_kernel(const __grid_constant__ PrefillArgs a,
                   const __grid_constant__ PrefillMaps maps) {
  using L = SlcLayout<D>;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* q_full = bars + 0;                    // [4]
  uint64_t* q_empty = bars + 4;                   // [4]
  uint64_t* k_full = bars + 8;                    // [kKSlots <= 8]
  uint64_t* k_empty = bars + 16;                  // [kKSlots]
  uint64_t* v_full = bars + 24;                   // [kVSlots <= 8]
  uint64_t* v_empty = bars + 32;                  // [kVSlots]
  uint64_t* s_full = bars + 40;                   // [2] TMEM score buffer per warpgroup
  uint64_t* s_empty = bars + 42;                  // [2]
  uint64_t* p_full = bars + 44;                   // [2] P^T buffer per warpgroup
  uint64_t* p_empty = bars + 46;                  // [2]
  uint64_t* o_full = bars + 48;                   // [4] output slots
  uint64_t* o_empty = bars + 52;                  // [4]
  uint64_t* fin = bars + 56;                      // [2] MMA drains
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 60);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 61);
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  float* inv_s = reinterpret_cast<float*>(sm + L::kInv);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (a.meta->bad) return;
  if (smem_u32(sm) & 1023u) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDeviceTimeoutCode);
    return;
  }
  // query slots start zeroed: with fewer than 16 query heads the MMA's 16
  // B rows reach past the loaded ones (their columns are never used)
  for (int i = threadIdx.x; i < L::kQSlots * L::kQBytes / 16; i += blockDim.x)
    reinterpret_cast<int4*>(sm + L::kQ)[i] = make_int4(0, 0, 0, 0);
  fence_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, 4);
    }
    for (int i = 0; i < L::kKSlots; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < L::kVSlots; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, 4);
      mbar_init(p_full + i, 4);
      mbar_init(p_empty + i, 1);
      mbar_init(fin + i, 1);
    }
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
  // selection blocks of l' tokens
  const int G = a.geo.G, l = a.geo.ls, lg_l = a.geo.lg_ls, n = a.geo.n;
  const int bpc = kChunk >> lg_l;        // blocks per 128-key chunk
  const int nsc = (n + bpc - 1) / bpc;   // chunks per job
  const int njobs = slc_jobs_of_cta(a);
  const int q_heads = a.geo.Hq < 16 ? a.geo.Hq : 16;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // The whole warp walks the jobs (lane i holds selection entry i, read one
    // job ahead); lane 0 waits on the ring and issues the copies.
    const bool is_k = warp == 0;
    if (lane == 0) {
      tma_prefetch_desc(is_k ? &maps.k_blk : (a.split_v ? &maps.v_split : &maps.v_blk));
      if (is_k) tma_prefetch_desc(a.split_q ? &maps.q_split : &maps.q_tok);
    }
    int slot_uses = 0;  // ring slots filled so far
    int qc = 0;
    const int nslots = is_k ? L::kKSlots : L::kVSlots;
    uint64_t* full = is_k ? k_full : v_full;
    uint64_t* empty = is_k ? k_empty : v_empty;
    bool ok = true;
    SlcJob nj = slc_job(a, blockIdx.x);
    int nidx = job_sel(a, nj, lane);
    for (int j = 0; j < njobs && ok; ++j) {
      const SlcJob job = nj;
      const int idx = nidx;
      nj = slc_job(a, blockIdx.x + (long long)(j + 1) * gridDim.x);
      nidx = job_sel(a, nj, lane);
      if (is_k) {
        const int qs = qc % L::kQSlots, u = qc / L::kQSlots;
        if (lane == 0) {
          if (u > 0 && !mbar_wait(q_empty + qs, (u - 1) & 1, abort_flag, status, kWaitCycles))
            ok = false;
          if (ok) {
            mbar_arrive_expect_tx(q_full + qs, q_heads * D * 2);
            if (a.split_q) {
              tma_load_4d(sm + L::kQ + qs * L::kQBytes, &maps.q_split, q_full + qs, 0, job.g * G,
                          0, job.row);
            } else {
#pragma unroll
              for (int h = 0; h < D / 64; ++h)
                tma_load_3d(sm + L::kQ + qs * L::kQBytes + h * 2048, &maps.q_tok, q_full + qs,
                            h * 64, job.g * G, job.row);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        ++qc;
      }
      // K: slot = (chunk c, channel half hh), bpc blocks of l keys each;
      // V: slot = (chunk c, 64-key half hv), 64 / l blocks x D channels.
      // Slots go in pairs: lane 0 claims both, then one lane per copy issues
      // (a thread streams one copy per few hundred cycles, so the copies of a
      // pair are spread over up to eight lanes).
      const int per_chunk = is_k ? D / 64 : 2;
      const int nblk = is_k ? bpc : (64 >> lg_l);       // blocks per slot
      const bool v_one = !is_k && a.split_v;            // one copy brings a whole V block
      const int cps = is_k ? nblk : (v_one ? 1 : nblk * (D / 64));  // copies per slot
      const int slots_per_job = nsc * per_chunk;
      for (int q0 = 0; q0 < slots_per_job && ok; q0 += 2) {
        const int ns = slots_per_job - q0 < 2 ? slots_per_job - q0 : 2;
        if (lane == 0) {
          for (int i = 0; i < ns && ok; ++i) {
            const int s = (slot_uses + i) % nslots, u = (slot_uses + i) / nslots;
            if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, abort_flag, status, kWaitCycles))
              ok = false;
            else
              mbar_arrive_expect_tx(full + s, is_k ? L::kKBytes : L::kVBytes);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        // copy `lane`: slot q0 + lane / cps, copy e = lane % cps of that slot
        const int qi = lane / cps, e = lane - qi * cps, q = q0 + qi;
        const int c = q / per_chunk, part = q - c * per_chunk;
        const int sub = is_k ? e : (v_one ? 0 : e / (D / 64));
        const int dh = is_k ? part : (v_one ? 0 : e - sub * (D / 64));
        const int bs = c * bpc + (is_k ? 0 : part * nblk) + sub;
        const int blk = __shfl_sync(0xffffffffu, idx, bs & 31);
        if (ok && qi < ns) {
          const int s = (slot_uses + qi) % nslots;
          const int row = (bs < n && blk >= 0) ? job.cu0 + (blk << lg_l) : -(1 << 24);
          if (is_k)
            tma_load_3d(sm + L::kK + s * L::kKBytes + sub * l * 128, &maps.k_blk, k_full + s,
                        dh * 64, job.g, row);
          else if (v_one)
            tma_load_4d(sm + L::kV + s * L::kVBytes, &maps.v_split, v_full + s, 0, row, 0, job.g);
          else
            tma_load_3d(sm + L::kV + s * L::kVBytes + dh * 8192 + sub * l * 128, &maps.v_blk,
                        v_full + s, dh * 64, job.g, row);
        }
        if (ok) slot_uses += ns;  // slots with copies in flight (drained below)
      }
    }
    // drain: every issued copy has landed before the CTA retires (also after
    // an abort, hence a private never-set abort flag)
    if (lane == 0) {
      volatile int never = 0;
      for (int s = 0; s < nslots && s < slot_uses; ++s) {
        const int last = slot_uses - 1 - ((slot_uses - 1 - s) % nslots);
        mbar_wait(full + s, (last / nslots) & 1, &never, nullptr, kWaitCycles / 4);
      }
      for (int qs = 0; qs < L::kQSlots && qs < qc; ++qs) {
        const int last = qc - 1 - ((qc - 1 - qs) % L::kQSlots);
        mbar_wait(q_full + qs, (last / L::kQSlots) & 1, &never, nullptr, kWaitCycles / 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK^T issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 16, false, false);
      int kc = 0;
      bool ok = true;
      for (int j = 0; j < njobs && ok; ++j) {
        const int qs = j % L::kQSlots, buf = j & 1, u = j >> 1;
        if (!mbar_wait(q_full + qs, (j / L::kQSlots) & 1, abort_flag, status, kWaitCycles) ||
            (u > 0 && !mbar_wait(s_empty + buf, (u - 1) & 1, abort_flag, status, kWaitCycles))) {
          ok = false;
          break;
        }
        const uint32_t qbuf = sbase + L::kQ + qs * L::kQBytes;
        for (int c = 0; c < nsc && ok; ++c) {
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh) {
            const int s = kc % L::kKSlots;
            if (!mbar_wait(k_full + s, (kc / L::kKSlots) & 1, abort_flag, status, kWaitCycles)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kslot = sbase + L::kK + s * L::kKBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(tmem + buf * 128 + c * 16,
                          smem_desc(kslot + kk * 32, 16, 1024, kLayoutSw128),
                          smem_desc(qbuf + hh * 2048 + kk * 32, 16, 1024, kLayoutSw128), id_qk,
                          (hh > 0 || kk > 0) ? 1u : 0u);
            mma_commit(k_empty + s);
            ++kc;
          }
        }
        if (!ok) break;
        mma_commit(s_full + buf);
        mma_commit(q_empty + qs);
      }
      mma_commit(fin + 0);
      volatile int never = 0;
      mbar_wait(fin + 0, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t id_pv = idesc_bf16(128, 16, true, true);
      int vc = 0;
      bool ok = true;
      for (int j = 0; j < njobs && ok; ++j) {
        const int buf = j & 1, os = j & 3;
        if (!mbar_wait(p_full + buf, (j >> 1) & 1, abort_flag, status, kWaitCycles) ||
            (j >= 4 && !mbar_wait(o_empty + os, ((j >> 2) - 1) & 1, abort_flag, status, kWaitCycles))) {
          ok = false;
          break;
        }
        const uint32_t P = sbase + L::kP + buf * L::kPBytes;
        for (int c = 0; c < nsc && ok; ++c) {
#pragma unroll
          for (int hv = 0; hv < 2; ++hv) {
            const int s = vc % L::kVSlots;
            if (!mbar_wait(v_full + s, (vc / L::kVSlots) & 1, abort_flag, status, kWaitCycles)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vslot = sbase + L::kV + s * L::kVBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(tmem + kColO + os * 16,
                          smem_desc(vslot + kk * 2048, 8192, 1024, kLayoutSw128),
                          smem_desc(P + c * 4096 + (hv * 4 + kk) * 256, 128, 2048, kLayoutNone),
                          id_pv, (c > 0 || hv > 0 || kk > 0) ? 1u : 0u);
            mma_commit(v_empty + s);
            ++vc;
          }
        }
        if (!ok) break;
        mma_commit(p_empty + buf);
        mma_commit(o_full + os);
      }
      mma_commit(fin + 1);
      volatile int never = 0;
      mbar_wait(fin + 1, 0, &never, nullptr, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int w = (warp - 4) >> 2;  // warpgroup: jobs j with j % 2 == w
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // key lane of every chunk; channel in the epilogue
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float sl2 = a.geo.scale_log2;
    const int Hq = a.geo.Hq, Hkv = a.geo.Hkv;
    const uint32_t colmask = G >= 16 ? 0xFFFFu : ((1u << G) - 1u);
    const int key_in_blk = r & (l - 1), slot_in_chunk = r >> lg_l;
    float* red_w = red + w * 128;

    // block of this thread's key in every chunk of job j (-1: none)
    auto load_blk = [&](const SlcJob& jb, int (&blk)[8]) {
      const int* sel = a.sel + ((size_t)jb.row * Hkv + jb.g) * n;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int bs = c * bpc + slot_in_chunk;
        blk[c] = (jb.valid && c < nsc && bs < n) ? __ldg(sel + bs) : -1;
      }
    };
    // output of job j (thread = channel r < D): g_cmp O_cmp + g_slc O_slc / sum + g_win O_win
    // (O_slc / sum alone in select-only block attention)
    auto epilogue = [&](int j) {
      const SlcJob jb = slc_job(a, blockIdx.x + (long long)j * gridDim.x);
      const int os = j & 3;
      float oc[16], ow[16], g0[16], g1[16];
      const bool gated = !a.select_only;  // select-only: out = O_slc
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const bool v = r < D && h < G;
        const bool vg = v && gated;
        const size_t gh = (size_t)jb.row * Hq + jb.g * G + h;
        oc[h] = vg ? a.o_cmp[gh * D + r] : 0.f;
        ow[h] = vg ? a.o_win[gh * D + r] : 0.f;
        g0[h] = vg ? __ldg(a.gates + gh * 3 + 0) : 0.f;
        g1[h] = vg ? __ldg(a.gates + gh * 3 + 1) : (v ? 1.f : 0.f);
      }
      mbar_wait(o_full + os, (j >> 2) & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      float o[16];
      tmem_ld16(lane_addr + kColO + os * 16, o);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty + os);
      if (r < D && !*abort_flag) {
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          if (h >= G) break;
          const float val = g0[h] * oc[h] + g1[h] * o[h] * inv_s[os * 16 + h] + ow[h];
          const size_t oi = ((size_t)jb.row * Hq + jb.g * G + h) * D + r;
          if (a.geo.out_f32) {
            static_cast<float*>(a.out)[oi] = val;
          } else {
            const __nv_bfloat16 bv = __float2bfloat16_rn(val);
            static_cast<uint16_t*>(a.out)[oi] = *reinterpret_cast<const uint16_t*>(&bv);
          }
        }
      }
    };

    int blk_next[8];
    SlcJob nj = slc_job(a, blockIdx.x + (long long)w * gridDim.x);
    load_blk(nj, blk_next);
    int k = 0;  // jobs of this warpgroup so far
    for (int j = w; j < njobs; j += 2, ++k) {
      const SlcJob jb = nj;
      uint32_t kok = 0;  // chunks whose key r is a visible selected key
#pragma unroll
      for (int c = 0; c < 8; ++c)
        kok |= (blk_next[c] >= 0 && (blk_next[c] << lg_l) + key_in_blk <= jb.t) ? (1u << c) : 0u;
      nj = slc_job(a, blockIdx.x + (long long)(j + 2) * gridDim.x);
      load_blk(nj, blk_next);
      // the epilogue of job j (one job from now) reads its G rows of O_cmp
      // and g_win O_win from HBM: bring them into L2 now, one 128-byte line
      // per thread (G * D * 4 bytes each)
      if (jb.valid && !a.select_only) {
        const size_t base = ((size_t)jb.row * Hq + jb.g * G) * D;
        const int lines = (G * D * 4) >> 7;
        if (r < lines) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.o_cmp + base + r * 32) : "memory");
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.o_win + base + r * 32) : "memory");
        }
      }

      mbar_wait(s_full + w, k & 1, abort_flag, status, kWaitCycles);
      tc_fence_after();
      // sweep 1: per-head maximum over this thread's keys
      float mx[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < 8; c0 += 4) {
        if (c0 >= nsc) break;
        float v[64];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float u16[16];
          tmem_ld16(lane_addr + w * 128 + (c0 + cc) * 16, u16);
#pragma unroll
          for (int h = 0; h < 16; ++h) v[cc * 16 + h] = u16[h];
        }
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if ((kok >> (c0 + cc)) & 1u) {
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], v[cc * 16 + h]);
          }
        }
      }
      if (w == 0) reduce16_across_128<1>(mx, red_w, q4, lane, true);
      else reduce16_across_128<2>(mx, red_w, q4, lane, true);
      float nmx[16];  // -max * scale: the exponent is one FFMA
#pragma unroll
      for (int h = 0; h < 16; ++h) nmx[h] = ((colmask >> h) & 1u) ? -mx[h] * sl2 : 0.f;
      // sweep 2: probabilities, per-head sums, P^T (bf16, largest element 1)
      if (k > 0) mbar_wait(p_empty + w, (k - 1) & 1, abort_flag, status, kWaitCycles);
      const uint32_t pbase = sbase + L::kP + w * L::kPBytes + (r >> 3) * 128 + (r & 7) * 16;
      float sum[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) sum[h] = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < 8; c0 += 4) {
        if (c0 >= nsc) break;
        float v[64];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float u16[16];
          tmem_ld16(lane_addr + w * 128 + (c0 + cc) * 16, u16);
#pragma unroll
          for (int h = 0; h < 16; ++h) v[cc * 16 + h] = u16[h];
        }
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = c0 + cc;
          if (c >= nsc) break;
          const bool on = (kok >> c) & 1u;
          float p[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            p[h] = (on && ((colmask >> h) & 1u)) ? ex2(fmaf(v[cc * 16 + h], sl2, nmx[h])) : 0.f;
            sum[h] += p[h];
          }
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) pk[q] = pack_bf16x2(p[2 * q], p[2 * q + 1]);
          st_shared_v4(pbase + c * 4096, pk[0], pk[1], pk[2], pk[3]);
          st_shared_v4(pbase + c * 4096 + 2048, pk[4], pk[5], pk[6], pk[7]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(s_empty + w);
        mbar_arrive(p_full + w);
      }
      if (w == 0) reduce16_across_128<1>(sum, red_w + 64, q4, lane, false);
      else reduce16_across_128<2>(sum, red_w + 64, q4, lane, false);
      // 1 / sum per head for the epilogue of this job (read one job later,
      // after this warpgroup's next named barrier)
      if (r < 16) {
        float sv = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h) sv = (h == r) ? sum[h] : sv;
        inv_s[(j & 3) * 16 + r] = (((colmask >> r) & 1u) && sv > 0.f) ? 1.f / sv : 0.f;
      }
      if (k > 0) epilogue(j - 2);
    }
    if (k > 0) {
      if (w == 0) named_bar_128<1>();
      else named_bar_128<2>();
      epilogue(w + 2 * (k - 1));
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
cudaError_t launch_slc_t(const PrefillArgs& a, const PrefillMaps& m, int num_sms,
                         cudaStream_t s) {
  using L = SlcLayout<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(nsa_slc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int grid = num_sms < kMaxPersistentCtas ? num_sms : kMaxPersistentCtas;
  nsa_slc_kernel<D><<<grid, kSlcThreads, L::kSmem, s>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_slc(const PrefillArgs& a, const PrefillMaps& m, int num_sms, cudaStream_t s) {
  return a.geo.D == 128 ? launch_slc_t<128>(a, m, num_sms, s)
                        : launch_slc_t<64>(a, m, num_sms, s);
}

}  // namespace nsa
