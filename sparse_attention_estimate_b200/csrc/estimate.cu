// estimate.cu - estimation of the vertical-slash pattern and the recall
// histogram of sparsity refinement, on tcgen05 tensor cores.
//
// Qwen2.5-1M explainer: "Sparse Attention" step 2 (attention of the last
// queries against all keys), "Chunked Prefill" (the last 64 queries of each
// chunk), "Algorithm" (selection with continuous positions), "Sparsity
// Refinement" (attention recall = exp(lse_sparse - lse_full)).
//
// One CTA handles one KV head's group (g query heads x 64 estimation rows,
// tiled as M = 128-row MMA tiles holding two heads each) over a contiguous
// range of 128-key blocks. Warp 0 issues TMA loads of rotated K blocks into a
// two-stage ring, warp 1 issues S = Q K^T (tcgen05.mma, M=128 N=128 K=16 bf16,
// fp32 accumulators in TMEM, one 128-column region per M tile), and two
// warpgroups (warps 4-7 and 8-11, each thread one TMEM lane = one query row)
// read S back with tcgen05.ld and run the epilogue of the pass:
//   kLse    running row max / sum of exp2 -> per-split partials, combined
//           afterwards into lse (natural log)
//   kSums   A = exp(s - lse); column sums (vertical) with a warp transpose-sum;
//           diagonal sums (slash) by rotating each lane's 32 values by its lane
//           index, splitting wrapped / unwrapped parts and transpose-summing
//           both; written as per-(head, 32-row half) partial arrays that a fixup
//           kernel adds in a fixed order (deterministic, no atomics)
//   kRecall A = exp(s - lse) added to every refinement level that selects the
//           element: the levels t >= min(its column's level, its offset's level),
//           so level t accumulates the recall mass of C_t directly
#include <algorithm>
#include <cmath>

#include "internal.cuh"

namespace vs {

enum EstMode { kLse = 0, kSums = 1, kRecall = 2 };
constexpr int kBinLevels = 16;  // recall levels binned in shared memory (the rest in registers)

constexpr int kEstThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSOff = 96;  // index offset of the slash partial arrays (skew >= -95)

struct EstParams {
  int64_t e;          // visible keys
  int64_t row0;       // position of estimation row 0 (= e - nr)
  int64_t e_pad;      // row stride of the partial arrays
  int nr;             // estimation rows per head
  int g, ntile, hq;
  int nblk;           // end of this launch's key-block range (blocks [blk0, nblk))
  int blk0;           // first key block of this launch
  int split0;         // index of this launch's first split in the partial outputs
  int bps;            // key blocks per split
  float scale_log2;   // softmax_scale * log2(e)
  float* part_ml;     // kLse: [nsplit][hq*64][2] (max, sum) in log2 units
  const float* lse;   // kSums / kRecall: [hq][64] natural log
  float* part_v;      // kSums: [hq][2][e_pad]
  float* part_s;      // kSums: [hq][2][2][e_pad + 256]
  const uint8_t* lvl; // kRecall: [hq][2][e_pad]
  float* hist;        // kRecall: [nsplit][hq][kMaxLevels]
  const int* dec;     // kRecall: heads already decided at the base budgets (nullable); a CTA
                      // whose g heads all are skips its pass
  int nlev;
  DevCommon dc;
};

struct __align__(1024) EstSmem {
  bf16 q[4][2][kTile * 64];  // [M tile][column half], 128-byte swizzled
  bf16 k[2][2][kTile * 64];  // [stage][column half]
  uint64_t q_full, k_full[2], k_empty[2], s_full[4], s_empty[4], drain;
  uint32_t tmem_base;
  int abort_word;
  float red[8][kRecallLevels];
  // kRecall: per-thread bins of the first kBinLevels levels, [warpgroup][M tile of
  // the thread][level][TMEM lane]; a thread owns its bins, and lane-major order puts
  // a warp's 32 bins of one level in 32 distinct banks
  float rbin[2][2][kBinLevels][kTile];
};

static_assert(sizeof(EstSmem) + 1024 <= 232448, "estimation shared memory exceeds 227 KB per CTA");

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Lane x ends with the sum over the warp's lanes of v[x] (v is consumed).
__device__ __forceinline__ float warp_transpose_sum32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float keep = upper ? v[i + s] : v[i];
      const float send = upper ? v[i] : v[i + s];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// v[i] <- v[(i + r) mod 32] for a per-lane r in [0, 32): five conditional rotations.
__device__ __forceinline__ void rotate_by(float (&v)[32], int r) {
#pragma unroll
  for (int b = 0; b < 5; ++b) {
    const bool on = (r >> b) & 1;
    const int sh = 1 << b;
    float t[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] = on ? v[(i + sh) & 31] : v[i];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = t[i];
  }
}

// Bounded wait that ignores the abort word (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit) break;
}

template <int MODE>
__global__ void __launch_bounds__(kEstThreads, 1)
    est_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               EstParams p) {
  extern __shared__ unsigned char smem_raw[];
  EstSmem& s = *reinterpret_cast<EstSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = blockIdx.y, split = p.split0 + static_cast<int>(blockIdx.x);
  if (MODE == kRecall && p.dec) {  // uniform over the CTA, before any barrier or allocation
    bool all = true;
    for (int hh = 0; hh < p.g; ++hh) all = all && p.dec[G * p.g + hh] != 0;
    if (all) return;
  }
  const int b_begin = p.blk0 + static_cast<int>(blockIdx.x) * p.bps;
  const int b_end = min(b_begin + p.bps, p.nblk);
  const int nb = b_end - b_begin;
  volatile int* abort_word = &s.abort_word;

  if (tid == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int t = 0; t < 4; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_empty[t], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort_word = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nb > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(&s.q_full, p.ntile * 2 * kTile * 64 * 2);
      for (int t = 0; t < p.ntile; ++t)
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(s.q[t][hf], &tmQ, &s.q_full, hf * 64, t * kTile, G);
      int issued[2] = {0, 0};
      bool ok = true;
      for (int i = 0; i < nb && ok; ++i) {
        const int st = i & 1;
        if (i >= 2) ok = mbar_wait(&s.k_empty[st], ((i >> 1) - 1) & 1, abort_word, p.dc.err);
        if (!ok) break;
        mbar_arrive_expect_tx(&s.k_full[st], 2 * kTile * 64 * 2);
        const int kb = b_begin + i;
        tma_load_3d(s.k[st][0], &tmK, &s.k_full[st], 0, kb * kTile, G);
        tma_load_3d(s.k[st][1], &tmK, &s.k_full[st], 64, kb * kTile, G);
        ++issued[st];
      }
      if (!ok) {  // let every issued copy land before the CTA exits
        drain_wait(&s.q_full, 0, p.dc.wait_ns);
        for (int st = 0; st < 2; ++st)
          if (issued[st] > 0) drain_wait(&s.k_full[st], (issued[st] - 1) & 1, p.dc.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nb > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      bool ok = mbar_wait(&s.q_full, 0, abort_word, p.dc.err);
      tc_fence_after_sync();
      for (int i = 0; i < nb && ok; ++i) {
        const int st = i & 1;
        ok = mbar_wait(&s.k_full[st], (i >> 1) & 1, abort_word, p.dc.err);
        if (!ok) break;
        tc_fence_after_sync();
        for (int t = 0; t < p.ntile && ok; ++t) {
          if (i >= 1) ok = mbar_wait(&s.s_empty[t], (i - 1) & 1, abort_word, p.dc.err);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t dt = tbase + t * kTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * (kTile * 64 * 2) + (kk & 3) * 32;
            const uint64_t da = smem_desc_sw128(smem_u32(&s.q[t][0][0]) + off, 16, 1024);
            const uint64_t db = smem_desc_sw128(smem_u32(&s.k[st][0][0]) + off, 16, 1024);
            mma_bf16_ss(dt, da, db, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s.s_full[t]);
        }
        mma_commit(&s.k_empty[st]);
      }
      // all issued MMAs complete before TMEM is released
      mma_commit(&s.drain);
      drain_wait(&s.drain, 0, p.dc.wait_ns);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue warpgroups
    const int wg = (warp - 4) >> 2;  // 0 or 1
    const int wl = warp & 3;         // TMEM lane quarter
    const int m = wl * 32 + lane;    // row within the M tile
    const int r = m & 63;            // estimation row within the head
    const int half = wl & 1;         // 32-row half of the head
    float st_m[2] = {-INFINITY, -INFINITY}, st_l[2] = {0.f, 0.f};
    float lse2[2] = {0.f, 0.f};
    float acc[2][kRecallLevels];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int t = 0; t < kRecallLevels; ++t) acc[a][t] = 0.f;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int t = wg + 2 * a;
      const int hh = 2 * t + (m >> 6);
      if (MODE != kLse && t < p.ntile && hh < p.g && r < p.nr)
        lse2[a] = p.lse[(G * p.g + hh) * kEstRows + r] * kLog2e;
    }
    if (MODE == kRecall) {
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int l = 0; l < kBinLevels; ++l) s.rbin[wg][a][l][m] = 0.f;
    }
    const int64_t irow = p.row0 + r;  // absolute position of this row
    bool ok = true;
    for (int i = 0; i < nb && ok; ++i) {
      const int kb = b_begin + i;
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int t = wg + 2 * a;
        if (t >= p.ntile) break;
        const int hh = 2 * t + (m >> 6);  // warp-uniform
        const bool head_ok = hh < p.g;
        const bool row_ok = head_ok && r < p.nr;
        const int h = G * p.g + hh;
        ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[t], i & 1, abort_word, p.dc.err));
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32];
          tmem_ld32(tmem_addr(tbase + t * kTile, wl * 32, c * 32), raw);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.s_empty[t]);
          }
          const int64_t j0 = static_cast<int64_t>(kb) * kTile + c * 32;
          float v[32];
          if (MODE == kLse) {
            float mx = -INFINITY;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const bool valid = row_ok && (j0 + x <= irow);
              v[x] = valid ? __uint_as_float(raw[x]) * p.scale_log2 : -INFINITY;
              mx = fmaxf(mx, v[x]);
            }
            const float mnew = fmaxf(st_m[a], mx);
            if (mnew != -INFINITY) {
              float sum = 0.f;
#pragma unroll
              for (int x = 0; x < 32; ++x) sum += ex2(v[x] - mnew);
              st_l[a] = st_l[a] * ex2(st_m[a] - mnew) + sum;
              st_m[a] = mnew;
            }
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const bool valid = row_ok && (j0 + x <= irow);
              v[x] = valid ? ex2(__uint_as_float(raw[x]) * p.scale_log2 - lse2[a]) : 0.f;
            }
            if (MODE == kSums) {
              if (head_ok) {
                // slash: lane l holds row r0 + l; rotate so register i holds column i + l
                float lo[32], hi[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) lo[x] = v[x];
                rotate_by(lo, lane);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                  const bool wrapped = x + lane >= 32;
                  hi[x] = wrapped ? lo[x] : 0.f;
                  lo[x] = wrapped ? 0.f : lo[x];
                }
                const float vs = warp_transpose_sum32(v);
                const float los = warp_transpose_sum32(lo);
                const float his = warp_transpose_sum32(hi);
                const int64_t r0 = half * 32;
                p.part_v[(static_cast<int64_t>(h) * 2 + half) * p.e_pad + j0 + lane] = vs;
                float* ps = p.part_s + (static_cast<int64_t>(h) * 2 + half) * 2 * (p.e_pad + 256);
                ps[j0 + lane - r0 + kSOff] = los;
                ps[(p.e_pad + 256) + j0 + lane - 32 - r0 + kSOff] = his;
              }
            } else {  // kRecall
              if (row_ok) {
                // An element selected first at level lv (the smaller of its column's and
                // its offset's level) belongs to every level t >= lv. Its probability goes
                // to bin lv (a plain shared-memory add: only this thread touches its bins,
                // and that measured faster than an atomic add); the bins are prefix-summed
                // over levels at the end. Levels at
                // or above kBinLevels (only with tiny base budgets) are accumulated
                // cumulatively in registers instead. Masked-out (j > irow) elements have
                // v = 0 and read a clamped, in-range offset.
                const uint8_t* lv_v = p.lvl + static_cast<int64_t>(h) * 2 * p.e_pad;
                const uint8_t* lv_s = lv_v + p.e_pad;
                const uint32_t nlev = static_cast<uint32_t>(p.nlev);
                float* bins = &s.rbin[wg][a][0][m];
                uint32_t vw[8];  // the 32 columns' vertical levels, 4 per word (same for all lanes)
#pragma unroll
                for (int q = 0; q < 8; ++q) vw[q] = __ldg(reinterpret_cast<const uint32_t*>(lv_v + j0) + q);
                auto bin_elements = [&](auto slash_level) {
#pragma unroll
                  for (int x = 0; x < 32; ++x) {
                    const uint32_t lvv = (vw[x >> 2] >> (8 * (x & 3))) & 0xFFu;
                    const uint32_t lvs = slash_level(x);
                    const uint32_t lv = lvv < lvs ? lvv : lvs;
                    if (lv < nlev) {
                      if (lv < static_cast<uint32_t>(kBinLevels)) {
                        bins[lv * kTile] += v[x];  // this thread's own bin: no atomic needed
                      } else {
#pragma unroll
                        for (int t2 = kBinLevels; t2 < kRecallLevels; ++t2)
                          if (static_cast<uint32_t>(t2) >= lv) acc[a][t2] += v[x];
                      }
                    }
                  }
                };
                // the offsets of this lane's 32 elements, irow - j0 - x, are the byte window
                // [dbase, dbase + 31] of the slash levels, read backwards: eight or nine
                // aligned words, funnel-shifted into place. Windows reaching below offset 0
                // (the chunk at the diagonal) read byte by byte with the offset clamped.
                const int64_t dbase = irow - j0 - 31;
                if (dbase >= 0) {
                  const uint32_t* wp = reinterpret_cast<const uint32_t*>(lv_s) + (dbase >> 2);
                  const uint32_t sh = 8u * static_cast<uint32_t>(dbase & 3);
                  uint32_t wv[9];
#pragma unroll
                  for (int q = 0; q < 8; ++q) wv[q] = __ldg(wp + q);
                  wv[8] = sh ? __ldg(wp + 8) : 0u;  // the window's last byte is dbase + 31 <= irow < e_pad
                  uint32_t aw[8];
#pragma unroll
                  for (int q = 0; q < 8; ++q) aw[q] = __funnelshift_r(wv[q], wv[q + 1], sh);
                  if (nlev < static_cast<uint32_t>(kBinLevels)) {
                    // Four elements per byte-SIMD step: columns 4q..4q+3 have their vertical
                    // levels in vw[q] and their offsets' levels, byte-reversed, in aw[7 - q];
                    // an element's level is the smaller one, and levels at or past nlev (never
                    // selected) all go to bin nlev, which no level reads: no branch per element.
                    const uint32_t cap4 = nlev * 0x01010101u;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                      const uint32_t l4 = __vminu4(__vminu4(vw[q], __byte_perm(aw[7 - q], 0u, 0x0123)), cap4);
#pragma unroll
                      for (int b = 0; b < 4; ++b) bins[((l4 >> (8 * b)) & 0xFFu) * kTile] += v[4 * q + b];
                    }
                  } else {
                    bin_elements([&](int x) { return (aw[(31 - x) >> 2] >> (8 * ((31 - x) & 3))) & 0xFFu; });
                  }
                } else {
                  bin_elements([&](int x) {
                    const int64_t d = irow - (j0 + x);
                    return static_cast<uint32_t>(__ldg(lv_s + (d >= 0 ? d : 0)));
                  });
                }
              }
            }
          }
        }
      }
    }
    // ---------------------------------------------------------- per-split outputs
    if (MODE == kLse) {
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int t = wg + 2 * a;
        const int hh = 2 * t + (m >> 6);
        if (t < p.ntile && hh < p.g && r < p.nr) {
          float* o = p.part_ml + ((static_cast<int64_t>(split) * p.hq + G * p.g + hh) * kEstRows + r) * 2;
          o[0] = st_m[a];
          o[1] = st_l[a];
        }
      }
    } else if (MODE == kRecall) {
      // this thread's bins (written by this thread only) as cumulative level sums
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        float run = 0.f;
#pragma unroll
        for (int l = 0; l < kBinLevels; ++l) {
          run += s.rbin[wg][a][l][m];
          acc[a][l] = run;
        }
#pragma unroll
        for (int l = kBinLevels; l < kRecallLevels; ++l) acc[a][l] += run;
      }
      // warp sums per level, then the two 32-row halves of each head in a fixed order
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int t = wg + 2 * a;
#pragma unroll
        for (int t2 = 0; t2 < kRecallLevels; ++t2) {
          float x = acc[a][t2];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
          acc[a][t2] = x;
        }
        // warps 2k and 2k+1 of a warpgroup hold the two halves of one head
        const int slot = (wg * 4 + wl);
        if (lane == 0)
          for (int t2 = 0; t2 < kRecallLevels; ++t2) s.red[slot][t2] = acc[a][t2];
        asm volatile("bar.sync %0, 128;" ::"r"(1 + wg));
        const int hh = 2 * t + (wl >> 1);
        if (t < p.ntile && hh < p.g && half == 0 && lane < kRecallLevels) {
          const float tot = s.red[slot][lane] + s.red[slot + 1][lane];
          p.hist[(static_cast<int64_t>(split) * p.hq + G * p.g + hh) * kMaxLevels + lane] = tot;
        }
        asm volatile("bar.sync %0, 128;" ::"r"(1 + wg));
      }
    }
  }
  // ------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 512);
  }
}

// lse_i = ln 2 * (max + log2(sum)) over the splits, in split order.
__global__ void lse_combine_kernel(const float* __restrict__ part_ml, int nsplit, int hq, int nr,
                                   float* __restrict__ lse) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= hq * kEstRows) return;
  const int r = idx % kEstRows;
  if (r >= nr) {
    lse[idx] = -INFINITY;
    return;
  }
  float mx = -INFINITY;
  for (int sp = 0; sp < nsplit; ++sp) mx = fmaxf(mx, part_ml[(static_cast<int64_t>(sp) * hq * kEstRows + idx) * 2]);
  float sum = 0.f;
  for (int sp = 0; sp < nsplit; ++sp) {
    const float* q = part_ml + (static_cast<int64_t>(sp) * hq * kEstRows + idx) * 2;
    if (q[0] != -INFINITY) sum += q[1] * exp2f(q[0] - mx);
  }
  lse[idx] = (mx + log2f(sum)) * 0.69314718055994531f;
}

// vert[j] = sum of the two 32-row halves; slash[d] = the four partial arrays at
// skew k = row0 - d (lo/hi parts of both halves), each read only where written.
__global__ void sums_fixup_kernel(const float* __restrict__ part_v, const float* __restrict__ part_s,
                                  int64_t e, int64_t row0, int64_t e_pad, int64_t cover,
                                  float* __restrict__ vert, float* __restrict__ slash, int64_t e_ld) {
  const int h = blockIdx.y;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= e) return;
  const float* pv = part_v + static_cast<int64_t>(h) * 2 * e_pad;
  vert[static_cast<int64_t>(h) * e_ld + j] = pv[j] + pv[e_pad + j];
  const int64_t d = j;
  const int64_t k = row0 - d;
  float acc = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float* ps = part_s + (static_cast<int64_t>(h) * 2 + half) * 2 * (e_pad + 256);
    const int64_t r0 = half * 32;
    // lo array covers skews [-r0, cover-1-r0]; hi covers [-32-r0, cover-33-r0]
    if (k >= -r0 && k <= cover - 1 - r0) acc += ps[k + kSOff];
    if (k >= -32 - r0 && k <= cover - 33 - r0) acc += ps[(e_pad + 256) + k + kSOff];
  }
  slash[static_cast<int64_t>(h) * e_ld + d] = acc;
}

// Recall of the base budgets (refinement level 0) per head, from the sums of the
// estimation pass: the rows' attention mass on the selected elements is the mass of the
// selected columns (their vertical sums) plus that of the selected offsets (their slash
// sums) minus the mass of the elements both select, which only these elements' scores
// give (one dot product each; few at the base budgets, most of them near the diagonal).
// A grid of (kBaseSplits, hq) CTAs takes one slice of the columns each, 4096 at a time:
// every thread scans 16 columns' level bytes at once, adds the selected sums and queues
// its selected vertical columns in shared memory; then each warp takes queued columns in
// turn, its lanes the estimation rows (r and r + 32), and subtracts exp(s - lse) of the
// rows whose offset is selected too. The CTAs' sums are added in a fixed order by
// recall_base_finish_kernel (the result does not depend on scheduling), which sets
// dec[h] = 1 when the recall reaches tau: the head then needs no histogram of the
// higher levels.
constexpr int kBaseBatch = 4096;  // columns per batch of the base-recall scan
__global__ void __launch_bounds__(256) recall_base_kernel(
    const float* __restrict__ vert, const float* __restrict__ slash, int64_t e_ld, int64_t e, int nr,
    const uint8_t* __restrict__ lvl, int64_t e_pad, const float* __restrict__ lse,
    const uint16_t* __restrict__ q_est, int ntile, const uint16_t* __restrict__ k_rot, int64_t k_rows, int g,
    float scale_log2, double* __restrict__ part) {
  __shared__ int32_t queue[kBaseBatch];
  __shared__ int nq;
  __shared__ double red[256];
  const int h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hk = h / g, hh = h % g;
  const uint8_t* lv_v = lvl + static_cast<int64_t>(h) * 2 * e_pad;  // 16-byte aligned rows
  const uint8_t* lv_s = lv_v + e_pad;
  const float* vr = vert + static_cast<int64_t>(h) * e_ld;
  const float* sr = slash + static_cast<int64_t>(h) * e_ld;
  const int64_t row0 = e - nr;
  const int64_t per = ((e + 15) / 16 + gridDim.x - 1) / gridDim.x * 16;  // columns per CTA
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t j1 = j0 + per < e ? j0 + per : e;
  // this lane's estimation rows, their lse (log2 units) and query rows (256-byte aligned)
  const uint16_t* qbase = q_est + (static_cast<int64_t>(hk) * ntile * kTile + hh * kEstRows) * kD;
  float lse2[2];
  for (int t = 0; t < 2; ++t) {
    const int r = lane + 32 * t;
    lse2[t] = r < nr ? lse[static_cast<int64_t>(h) * kEstRows + r] * kLog2e : 0.f;
  }
  double acc = 0.0;  // vertical + slash - both
  for (int64_t rb = j0; rb < j1; rb += kBaseBatch) {
    if (tid == 0) nq = 0;
    __syncthreads();
    const int64_t jb = rb + 16 * tid;
    if (jb < j1) {
      const uint4 wv = *reinterpret_cast<const uint4*>(lv_v + jb);
      const uint4 ws = *reinterpret_cast<const uint4*>(lv_s + jb);
      const uint32_t av[4] = {wv.x, wv.y, wv.z, wv.w}, as[4] = {ws.x, ws.y, ws.z, ws.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // a zero byte is an element of the base level; most words hold none
        const uint32_t zv = __vcmpeq4(av[q], 0u), zs = __vcmpeq4(as[q], 0u);
        if ((zv | zs) == 0u) continue;
        for (int b = 0; b < 4; ++b) {
          const int64_t j = jb + 4 * q + b;
          if (j >= j1) break;
          if ((zs >> (8 * b)) & 1u) acc += sr[j];
          if ((zv >> (8 * b)) & 1u) {
            acc += vr[j];
            queue[atomicAdd(&nq, 1)] = static_cast<int32_t>(j - rb);
          }
        }
      }
    }
    __syncthreads();
    const int n = nq;
    for (int i = warp; i < n; i += 8) {
      const int64_t j = rb + queue[i];
      const uint4* kj = reinterpret_cast<const uint4*>(k_rot + (static_cast<int64_t>(hk) * k_rows + j) * kD);
      for (int t = 0; t < 2; ++t) {
        const int r = lane + 32 * t;
        const int64_t d = row0 + r - j;  // this element's offset
        if (r >= nr || d < 0 || lv_s[d] != 0) continue;
        const uint4* qr = reinterpret_cast<const uint4*>(qbase + static_cast<int64_t>(r) * kD);
        float dot = 0.f;
#pragma unroll 4
        for (int c = 0; c < kD / 8; ++c) {
          const uint4 a = qr[c], b = kj[c];
          const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            dot = fmaf(__uint_as_float(aw[u] << 16), __uint_as_float(bw[u] << 16), dot);
            dot = fmaf(__uint_as_float(aw[u] & 0xFFFF0000u), __uint_as_float(bw[u] & 0xFFFF0000u), dot);
          }
        }
        acc -= exp2f(dot * scale_log2 - lse2[t]);
      }
    }
    __syncthreads();  // the queue is refilled by the next batch
  }
  red[tid] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  if (tid == 0) part[static_cast<int64_t>(h) * gridDim.x + blockIdx.x] = red[0];
}

__global__ void recall_base_finish_kernel(const double* __restrict__ part, int nsplit, int hq, int nr,
                                          float tau, float* __restrict__ rc0, int* __restrict__ dec) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= hq) return;
  double sum = 0.0;
  for (int i = 0; i < nsplit; ++i) sum += part[static_cast<int64_t>(h) * nsplit + i];
  const float rc = static_cast<float>(sum / nr);
  rc0[h] = rc;
  dec[h] = rc >= tau ? 1 : 0;
}

vs_status run_recall_base(vs_ctx* c, const float* vert, const float* slash, int64_t e_ld, int64_t e, int nr,
                          const float* lse, float tau, cudaStream_t st) {
  const int hq = c->cfg.hq;
  double* part = ws_ptr<double>(c, c->L.base_part);
  recall_base_kernel<<<dim3(kBaseSplits, hq), 256, 0, st>>>(
      vert, slash, e_ld, e, nr, ws_ptr<uint8_t>(c, c->L.lvl), c->L.e_pad, lse,
      ws_ptr<uint16_t>(c, c->L.q_est), c->L.ntile, ws_ptr<uint16_t>(c, c->L.k_cont), c->max_seq,
      hq / c->cfg.hkv, c->cfg.softmax_scale * kLog2e, part);
  vs_status s = launched("recall_base_kernel launch");
  if (s != VS_OK) return s;
  recall_base_finish_kernel<<<(hq + 127) / 128, 128, 0, st>>>(
      part, kBaseSplits, hq, nr, tau, ws_ptr<float>(c, c->L.base_rc), ws_ptr<int>(c, c->L.base_rc) + hq);
  return launched("recall_base_finish_kernel launch");
}

// One estimation-kernel launch over key blocks [blk0, blk1) with the rotated rows
// in q_buf and the rotated keys in k_buf; its splits write partial outputs from
// index split0 on. *nsplit_out gets the number of splits used.
static vs_status launch_est_range(vs_ctx* c, int mode, int64_t e, int nr, const float* lse, int nlev,
                                  int blk0, int blk1, int split0, int max_splits, size_t q_buf,
                                  size_t k_buf, int* nsplit_out, cudaStream_t st, const int* dec = nullptr) {
  const int hkv = c->cfg.hkv, g = c->cfg.hq / c->cfg.hkv;
  const int nblk = blk1 - blk0;
  if (nblk <= 0) {
    *nsplit_out = 0;
    return VS_OK;
  }
  int nsplit = std::max(1, c->num_sms / hkv);
  nsplit = std::min(nsplit, nblk);
  nsplit = std::min(nsplit, max_splits);
  const int bps = static_cast<int>(ceil_div(nblk, nsplit));
  nsplit = static_cast<int>(ceil_div(nblk, bps));
  *nsplit_out = nsplit;
  CUtensorMap tmQ, tmK;
  vs_status s = make_tmap_rows(&tmQ, c->ws + q_buf, hkv, static_cast<int64_t>(c->L.ntile) * kTile,
                               static_cast<int64_t>(c->L.ntile) * kTile, kTile);
  if (s != VS_OK) return s;
  s = make_tmap_rows(&tmK, c->ws + k_buf, hkv, e, c->max_seq, kTile);
  if (s != VS_OK) return s;
  EstParams p{};
  p.e = e;
  p.row0 = e - nr;
  p.e_pad = c->L.e_pad;
  p.nr = nr;
  p.g = g;
  p.ntile = c->L.ntile;
  p.hq = c->cfg.hq;
  p.nblk = blk1;
  p.blk0 = blk0;
  p.split0 = split0;
  p.bps = bps;
  p.scale_log2 = c->cfg.softmax_scale * kLog2e;
  p.part_ml = ws_ptr<float>(c, c->L.est_ml);
  p.lse = lse;
  p.part_v = ws_ptr<float>(c, c->L.part_v);
  p.part_s = ws_ptr<float>(c, c->L.part_s);
  p.lvl = ws_ptr<uint8_t>(c, c->L.lvl);
  p.hist = ws_ptr<float>(c, c->L.hist);
  p.dec = dec;
  p.nlev = nlev;
  p.dc = dev_common(c);
  const size_t smem = sizeof(EstSmem) + 1024;
  dim3 grid(nsplit, hkv);
  if (mode == kLse) {
    cudaFuncSetAttribute(est_kernel<kLse>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    est_kernel<kLse><<<grid, kEstThreads, smem, st>>>(tmQ, tmK, p);
  } else if (mode == kSums) {
    cudaFuncSetAttribute(est_kernel<kSums>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    est_kernel<kSums><<<grid, kEstThreads, smem, st>>>(tmQ, tmK, p);
  } else {
    cudaFuncSetAttribute(est_kernel<kRecall>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    est_kernel<kRecall><<<grid, kEstThreads, smem, st>>>(tmQ, tmK, p);
  }
  return launched("est_kernel launch");
}

// All key blocks of [0, e) with continuous positions (estimation rows in q_est,
// keys in the continuous rotated cache).
static vs_status launch_est(vs_ctx* c, int mode, int64_t e, int nr, const float* lse, int nlev,
                            int* nsplit_out, cudaStream_t st, const int* dec = nullptr) {
  return launch_est_range(c, mode, e, nr, lse, nlev, 0, static_cast<int>(ceil_div(e, kTile)), 0,
                          c->L.nsplit_max, c->L.q_est, c->L.k_cont, nsplit_out, st, dec);
}

vs_status run_estimate(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                       const uint16_t* k, int64_t k_rows, int64_t e, float* vert, float* slash,
                       int64_t e_ld, float* lse, cudaStream_t st) {
  (void)q;
  (void)q_rows;
  (void)k;
  (void)k_rows;
  const int nr = static_cast<int>(e - std::max(q_pos0, e - static_cast<int64_t>(c->cfg.last_q)));
  int nsplit = 0;
  vs_status s = launch_est(c, kLse, e, nr, nullptr, 0, &nsplit, st);
  if (s != VS_OK) return s;
  const int n = c->cfg.hq * kEstRows;
  lse_combine_kernel<<<ceil_div(n, 256), 256, 0, st>>>(ws_ptr<float>(c, c->L.est_ml), nsplit,
                                                      c->cfg.hq, nr, lse);
  s = launched("lse_combine_kernel launch");
  if (s != VS_OK) return s;
  s = launch_est(c, kSums, e, nr, lse, 0, &nsplit, st);
  if (s != VS_OK) return s;
  const int64_t cover = ceil_div(e, kTile) * kTile;
  sums_fixup_kernel<<<dim3(static_cast<unsigned>(ceil_div(e, 256)), c->cfg.hq), 256, 0, st>>>(
      ws_ptr<float>(c, c->L.part_v), ws_ptr<float>(c, c->L.part_s), e, e - nr, c->L.e_pad, cover,
      vert, slash, e_ld);
  return launched("sums_fixup_kernel launch");
}

// The recall histogram from the estimation rows' attention at DCA positions (the
// attention the prefill computes) instead of continuous ones. The rows R lie in one
// DCA chunk b, so each 128-key block has one class for all of them (S % 128 == 0):
// keys in chunk b are intra, in chunk b-1 successive, before that inter. Per class,
// the rows are rotated at that class's query positions and the kernel runs over the
// class's key blocks against the DCA-rotated keys: first the lse pass (combined over
// all classes' splits), then the histogram pass with that lse.
vs_status run_recall_hist_dca(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                              const uint16_t* k, int64_t k_rows, int64_t e, int nr, int nlev,
                              cudaStream_t st) {
  const int64_t S = c->dca.S;
  VS_REQUIRE(S % kTile == 0, VS_ERR_UNSUPPORTED,
             "recall at DCA positions needs the DCA stride C - W to be a multiple of 128");
  const int64_t b = (e - 1) / S;
  VS_REQUIRE((e - nr) / S == b, VS_ERR_UNSUPPORTED,
             "the estimation rows straddle a DCA chunk boundary");
  VS_TRY(ensure_keys_rotated(c, k, k_rows, e, true, st));
  const int nblk = static_cast<int>(ceil_div(e, kTile));
  int lo[3], hi[3];  // key-block ranges by class: 0 intra, 1 successive, 2 inter
  lo[2] = 0;
  hi[2] = b >= 2 ? static_cast<int>((b - 1) * S / kTile) : 0;
  lo[1] = hi[2];
  hi[1] = b >= 1 ? static_cast<int>(b * S / kTile) : 0;
  lo[0] = hi[1];
  hi[0] = nblk;
  const int g = c->cfg.hq / c->cfg.hkv;
  auto rotate = [&](int cls) {
    return launch_rope_rows(c, reinterpret_cast<const bf16*>(q), q_rows, e - nr - q_pos0,
                            ws_ptr<bf16>(c, c->L.q_est), 0, 0, g,
                            static_cast<int64_t>(c->L.ntile) * kTile, kEstRows, nr, c->cfg.hq,
                            e - nr, 2 + cls, st);
  };
  float* lse_dca = ws_ptr<float>(c, c->L.lse_dca);
  int total[2] = {0, 0};
  for (int pass = 0; pass < 2; ++pass) {
    for (int cls = 2; cls >= 0; --cls) {
      if (hi[cls] <= lo[cls]) continue;
      VS_TRY(rotate(cls));
      const int budget = std::max(1, (c->L.nsplit_max - total[pass]) / (cls + 1));
      int ns = 0;
      VS_TRY(launch_est_range(c, pass == 0 ? kLse : kRecall, e, nr, pass == 0 ? nullptr : lse_dca,
                              pass == 0 ? 0 : nlev, lo[cls], hi[cls], total[pass], budget,
                              c->L.q_est, c->L.k_dca, &ns, st));
      total[pass] += ns;
    }
    if (pass == 0) {
      const int n = c->cfg.hq * kEstRows;
      lse_combine_kernel<<<ceil_div(n, 256), 256, 0, st>>>(ws_ptr<float>(c, c->L.est_ml), total[0],
                                                          c->cfg.hq, nr, lse_dca);
      VS_TRY(launched("lse_combine_kernel launch"));
    }
  }
  c->hist_nsplit = total[1];
  return VS_OK;
}

vs_status run_recall_hist(vs_ctx* c, int64_t e, int nr, const float* lse, int nlev,
                          cudaStream_t st, const int* dec) {
  int nsplit = 0;
  vs_status s = launch_est(c, kRecall, e, nr, lse, nlev, &nsplit, st, dec);
  c->hist_nsplit = nsplit;
  return s;
}

}  // namespace vs
