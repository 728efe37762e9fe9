// attn.cu - vertical-slash sparse attention over one prefill chunk, on tcgen05.
//
// Qwen2.5-1M explainer: "Sparse Attention" step 4 (attention over the selected
// tokens only), "Algorithm" (attention with DCA positions; chunk rows attend the
// growing KV cache), "Length Extrapolation" (the three DCA patterns). The
// online-softmax tiling follows the FlashAttention framing of the long-context
// essay (section 3.2): no N x N matrix is materialised.
//
// Element mask: query row i sees key j iff j <= i and (j is a selected vertical
// column or i - j is a selected slash offset). Work is organised per CTA as one
// head and two adjacent 128-row query tiles; the key axis is cut into 128-key
// blocks, and a schedule kernel lists, per CTA, the blocks in which either tile
// has a selected element, tagging each (tile, block) as skip / partial / full.
//
// The attention kernel (one CTA per SM, 12 warps; after the role split the control
// warpgroup keeps 112 registers per thread and the softmax warpgroups 192):
//  warp 0     TMA producer: the two Q tiles (re-loaded with another rotation
//             when the DCA class of the key block changes), K and V blocks into
//             two-stage rings.
//  warp 1     MMA issuer (one thread): S_t = Q_t K^T (SS, M=128 N=128), then
//             O_t += P_t V (TS: P read from tensor memory, V MN-major in smem).
//  warps 4-7  softmax of tile 0, warps 8-11 of tile 1; one thread per query row:
//             tcgen05.ld of S, element mask from the vertical / slash bitmaps,
//             online softmax in fp32 with exp2, optimistic (a row with a reference
//             max skips the max pass unless the block's sum exceeds 2^16) and a lazy
//             rescale of O (only when the running max grows by more than 2^8), P as
//             bf16 written back into S's tensor-memory columns.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512); P_t aliases the first 64 columns of S_t. The next S_t MMA is
// issued after the PV MMA that reads P_t; tcgen05 MMAs of one thread execute in
// issue order.
#include <algorithm>
#include <cmath>

#include "internal.cuh"

namespace vs {

constexpr int kAttnThreads = 384;
// Register budgets after the role split: warpgroup 0 (TMA producer, MMA issuer, two
// idle warps) keeps 112 per thread, the two softmax warpgroups take 192 each:
// 128 x 112 + 256 x 192 = 63488 <= 384 x 168 (the launch's 64512).
constexpr uint32_t kRegsControl = 112, kRegsSoftmax = 192;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= 384 * 168, "register split exceeds the launch");
constexpr float kLog2eA = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// A block exponentiated against the row's reference max without a max pass is kept
// when its row sum stays at or below this (every p <= 2^16, far inside bf16 and the
// fp32 accumulators); otherwise it is redone with its own max.
constexpr float kOptimisticSum = 65536.0f;
constexpr int kDevErrIndex = 4;            // an index list held an out-of-range entry

// ---------------------------------------------------------------- bitmaps
__global__ void set_bits_kernel(const int32_t* __restrict__ v_idx, int32_t cap_v,
                                const int32_t* __restrict__ v_cnt, const int32_t* __restrict__ s_off,
                                int32_t cap_s, const int32_t* __restrict__ s_cnt, int64_t e,
                                uint32_t* vbits, uint32_t* sbits, int64_t nwords, int* err) {
  const int h = blockIdx.y;
  const int arr = blockIdx.z;
  const int32_t cnt_raw = arr == 0 ? v_cnt[h] : s_cnt[h];
  const int32_t cap = arr == 0 ? cap_v : cap_s;
  const int32_t cnt = cnt_raw < 0 ? 0 : (cnt_raw > cap ? cap : cnt_raw);
  if (cnt_raw > cap && blockIdx.x == 0 && threadIdx.x == 0) atomicCAS(err, 0, kDevErrIndex);
  const int32_t* list = (arr == 0 ? v_idx + static_cast<int64_t>(h) * cap_v
                                  : s_off + static_cast<int64_t>(h) * cap_s);
  uint32_t* bits = (arr == 0 ? vbits : sbits) + static_cast<int64_t>(h) * nwords + (arr == 0 ? 0 : kSPad);
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; n < cnt;
       n += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = list[n];
    if (j < 0 || j >= e) {
      atomicCAS(err, 0, kDevErrIndex);
      continue;
    }
    atomicOr(bits + (j >> 5), 1u << (j & 31));
  }
}

// scum[h][w] = set bits of the slash bitmap in words [0, w)
__global__ void __launch_bounds__(1024) prefix_popc_kernel(const uint32_t* __restrict__ sbits,
                                                           int64_t nwords, uint32_t* scum) {
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t* b = sbits + static_cast<int64_t>(h) * nwords;
  uint32_t* o = scum + static_cast<int64_t>(h) * (nwords + 1);
  __shared__ uint32_t wsum[32];
  uint32_t running = 0;
  for (int64_t i0 = 0; i0 < nwords; i0 += 1024) {
    const int64_t i = i0 + tid;
    const uint32_t v = i < nwords ? __popc(b[i]) : 0u;
    uint32_t x = v;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, s);
      if (lane >= s) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
      uint32_t t = wsum[lane];
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, t, s);
        if (lane >= s) t += y;
      }
      wsum[lane] = t;
    }
    __syncthreads();
    const uint32_t excl = running + (w > 0 ? wsum[w - 1] : 0u) + x - v;
    if (i < nwords) o[i] = excl;
    running += wsum[31];
    __syncthreads();
  }
  if (tid == 0) o[nwords] = running;
}

// ---------------------------------------------------------------- schedule
__device__ __forceinline__ uint32_t bit_prefix(const uint32_t* bits, const uint32_t* cum, int64_t x) {
  const int64_t w = x >> 5;
  const int r = static_cast<int>(x & 31);
  return cum[w] + (r ? __popc(bits[w] & ((1u << r) - 1u)) : 0u);
}

// State of (query tile starting at R0, key block starting at k0): 0 skip, 1 partial, 2 full.
__device__ __forceinline__ int tile_block_state(int64_t R0, int64_t k0, int64_t e,
                                                const uint32_t* vb, const uint32_t* sb,
                                                const uint32_t* sc) {
  if (R0 >= e || k0 > R0 + 127) return 0;
  const int64_t dhi_raw = R0 + 127 - k0;
  const int64_t dlo = R0 - k0 - 127 > 0 ? R0 - k0 - 127 : 0;
  const int64_t dhi = dhi_raw < e - 1 ? dhi_raw : e - 1;
  uint32_t scount = 0;
  if (dhi >= dlo)
    scount = bit_prefix(sb, sc, dhi + 1 + 32 * kSPad) - bit_prefix(sb, sc, dlo + 32 * kSPad);
  const bool s_all = dhi >= dlo && scount == static_cast<uint32_t>(dhi - dlo + 1);
  const uint4 v = *reinterpret_cast<const uint4*>(vb + (k0 >> 5));
  const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
  const bool v_all = (v.x & v.y & v.z & v.w) == 0xFFFFFFFFu;
  const int64_t lim = dhi_raw;  // columns c <= lim can be causal for some row
  bool v_any = false;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t m;
    if (lim >= 32 * q + 31)
      m = 0xFFFFFFFFu;
    else if (lim < 32 * q)
      m = 0u;
    else
      m = (2u << (lim - 32 * q)) - 1u;
    v_any |= (vw[q] & m) != 0u;
  }
  if (v_all || s_all) return 2;
  return (v_any || scount > 0) ? 1 : 0;
}

__global__ void __launch_bounds__(256) schedule_kernel(
    const uint32_t* __restrict__ vbits, const uint32_t* __restrict__ sbits,
    const uint32_t* __restrict__ scum, int64_t nwords, int64_t q_pos0, int64_t e, int npairs_ws,
    int64_t nblk_ws, int32_t* __restrict__ sched, int32_t* __restrict__ sched_cnt,
    unsigned long long* stats) {
  const int pair = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t* vb = vbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sb = sbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sc = scum + static_cast<int64_t>(h) * (nwords + 1);
  const int64_t R0 = q_pos0 + static_cast<int64_t>(pair) * 256;
  const int64_t last_row = (e - 1 < R0 + 255) ? e - 1 : R0 + 255;
  const int64_t nb = last_row / kTile + 1;
  int32_t* out = sched + (static_cast<int64_t>(h) * npairs_ws + pair) * nblk_ws;
  __shared__ int wsum[8];
  int running = 0;
  for (int64_t b0 = 0; b0 < nb; b0 += 256) {
    const int64_t b = b0 + tid;
    int flags = 0;
    if (b < nb) {
      const int64_t k0 = b * kTile;
      flags = tile_block_state(R0, k0, e, vb, sb, sc) | (tile_block_state(R0 + 128, k0, e, vb, sb, sc) << 2);
    }
    const int f = flags != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[w] = __popc(bal);
    __syncthreads();
    int base = running;
    for (int i = 0; i < w; ++i) base += wsum[i];
    int total = 0;
    for (int i = 0; i < 8; ++i) total += wsum[i];
    if (f) out[base + __popc(bal & ((1u << lane) - 1u))] = static_cast<int32_t>(b) | (flags << 24);
    running += total;
    __syncthreads();
  }
  if (tid == 0) {
    sched_cnt[static_cast<int64_t>(h) * npairs_ws + pair] = running;
    atomicAdd(stats, 2ull * static_cast<unsigned long long>(running));
  }
}

// ---------------------------------------------------------------- attention
struct AttnParams {
  int64_t q_pos0, e;
  int hq, g, npairs;
  int nvar;
  float scale_log2;
  const int32_t* sched;
  const int32_t* sched_cnt;
  int npairs_ws;
  int64_t nblk_ws;
  const uint32_t* vbits;
  const uint32_t* sbits;
  int64_t nwords;
  uint16_t* out;
  int64_t out_rows;
  float* lse_out;
  unsigned long long* stats;
  DcaParams dca;
  DevCommon dc;
};

struct __align__(1024) AttnSmem {
  bf16 q[2][2][kTile * 64];  // [tile][column half]
  bf16 k[2][2][kTile * 64];  // [stage][column half]
  bf16 v[2][2][kTile * 64];  // [stage][column half]: 128 keys x 64 dims each
  uint64_t q_full[2], q_empty[2], k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_final, drain;
  uint32_t tmem_base;
  int abort_word;
};

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void drain_wait_a(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit) break;
}

// DCA class of (query tile starting at R0, key block starting at k0): 0 intra,
// 1 successive, 2 inter (always 0 without DCA).
__device__ __forceinline__ int dca_class(int64_t R0, int64_t k0, const DcaParams& d) {
  if (!d.enabled) return 0;
  const int64_t bi = R0 / d.S, bj = k0 / d.S;
  return bi == bj ? 0 : (bi == bj + 1 ? 1 : 2);
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  AttnSmem& s = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Work order: the KV groups one after another; inside a group the query-tile pairs
  // longest first, the g heads of a pair adjacent. The CTAs resident at any time then
  // belong to one KV head (two at a group boundary) and start together, so they sweep
  // its K/V blocks nearly in step and share each block through L2; with the heads of
  // all groups interleaved, a chunk's K/V (up to 4.3 GB at 1M keys) was re-read from HBM.
  const int per_group = p.npairs * p.g;
  const int hk = static_cast<int>(blockIdx.x) / per_group;
  const int rg = static_cast<int>(blockIdx.x) % per_group;
  const int pair = p.npairs - 1 - rg / p.g;
  const int h = hk * p.g + rg % p.g;
  const int64_t R0 = p.q_pos0 + static_cast<int64_t>(pair) * 256;  // tile 0's first row
  const int32_t* list = p.sched + (static_cast<int64_t>(h) * p.npairs_ws + pair) * p.nblk_ws;
  const int n = p.sched_cnt[static_cast<int64_t>(h) * p.npairs_ws + pair];
  volatile int* abort_word = &s.abort_word;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.q_full[i], 1);
      mbar_init(&s.q_empty[i], 1);
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 4);
    }
    mbar_init(&s.o_final, 1);
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
  constexpr uint32_t kTileBytes = kTile * 64 * 2;  // one 128 x 64 bf16 box
  if (warp < 4) {
    // warpgroup 0: the TMA producer (warp 0), the MMA issuer (warp 1), two idle warps
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && n > 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int cls[2];
        int qchg[2] = {0, 0};
        const int64_t kb0 = static_cast<int64_t>(list[0] & 0xFFFFFF) * kTile;
        for (int t = 0; t < 2; ++t) {
          cls[t] = dca_class(R0 + t * kTile, kb0, p.dca);
          mbar_arrive_expect_tx(&s.q_full[t], 2 * kTileBytes);
          const int qrow = pair * 256 + t * kTile;
          const int qh = cls[t] * p.hq + h;
          tma_load_3d(s.q[t][0], &tmQ, &s.q_full[t], 0, qrow, qh);
          tma_load_3d(s.q[t][1], &tmQ, &s.q_full[t], 64, qrow, qh);
        }
        int kiss[2] = {0, 0}, viss[2] = {0, 0};
        bool ok = true;
        int32_t ent = list[0];  // schedule entries are read one block ahead of use
        for (int j = 0; j < n && ok; ++j) {
          const int b = ent & 0xFFFFFF;
          ent = j + 1 < n ? ld_keep_s32(list + j + 1) : 0;
          const int st = j & 1;
          // K(j) first: the MMA warp releases a Q tile only after issuing S0(j)
          if (j >= 2) ok = mbar_wait(&s.k_empty[st], ((j >> 1) - 1) & 1, abort_word, p.dc.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&s.k_full[st], 2 * kTileBytes);
          tma_load_3d(s.k[st][0], &tmK, &s.k_full[st], 0, b * kTile, hk);
          tma_load_3d(s.k[st][1], &tmK, &s.k_full[st], 64, b * kTile, hk);
          ++kiss[st];
          if (j > 0) {
            for (int t = 0; t < 2 && ok; ++t) {
              const int c = dca_class(R0 + t * kTile, static_cast<int64_t>(b) * kTile, p.dca);
              if (c != cls[t]) {
                ok = mbar_wait(&s.q_empty[t], qchg[t] & 1, abort_word, p.dc.err);
                if (!ok) break;
                ++qchg[t];
                cls[t] = c;
                mbar_arrive_expect_tx(&s.q_full[t], 2 * kTileBytes);
                const int qrow = pair * 256 + t * kTile;
                tma_load_3d(s.q[t][0], &tmQ, &s.q_full[t], 0, qrow, c * p.hq + h);
                tma_load_3d(s.q[t][1], &tmQ, &s.q_full[t], 64, qrow, c * p.hq + h);
              }
            }
            if (!ok) break;
          }
          if (j >= 2) ok = mbar_wait(&s.v_empty[st], ((j >> 1) - 1) & 1, abort_word, p.dc.err);
          if (!ok) break;
          mbar_arrive_expect_tx(&s.v_full[st], 2 * kTileBytes);
          tma_load_3d(s.v[st][0], &tmV, &s.v_full[st], 0, b * kTile, hk);
          tma_load_3d(s.v[st][1], &tmV, &s.v_full[st], 64, b * kTile, hk);
          ++viss[st];
        }
        if (!ok) {  // let every issued copy land before the CTA exits
          for (int t = 0; t < 2; ++t) drain_wait_a(&s.q_full[t], qchg[t] & 1, p.dc.wait_ns);
          for (int st = 0; st < 2; ++st) {
            if (kiss[st] > 0) drain_wait_a(&s.k_full[st], (kiss[st] - 1) & 1, p.dc.wait_ns);
            if (viss[st] > 0) drain_wait_a(&s.v_full[st], (viss[st] - 1) & 1, p.dc.wait_ns);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        if (n > 0) {
          const uint32_t id_qk = idesc_bf16_f32(128, 128, 0, 0);
          const uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
          const uint32_t tS[2] = {tbase, tbase + 128};
          const uint32_t tO[2] = {tbase + 256, tbase + 384};
          int cls[2], qph[2] = {1, 1};
          const int64_t kb0 = static_cast<int64_t>(list[0] & 0xFFFFFF) * kTile;
          cls[0] = dca_class(R0, kb0, p.dca);
          cls[1] = dca_class(R0 + kTile, kb0, p.dca);
          int32_t ent1 = n > 1 ? list[1] : 0;  // entry of block j + 1, read a block ahead
          // descriptor words of the operand tiles (K-major Q and K, MN-major V; 128-byte swizzle)
          const uint32_t dhi = smem_desc_sw128_hi(1024);
          const uint32_t qlo[2] = {smem_desc_sw128_lo(smem_u32(&s.q[0][0][0]), 16),
                                   smem_desc_sw128_lo(smem_u32(&s.q[1][0][0]), 16)};
          const uint32_t klo[2] = {smem_desc_sw128_lo(smem_u32(&s.k[0][0][0]), 16),
                                   smem_desc_sw128_lo(smem_u32(&s.k[1][0][0]), 16)};
          const uint32_t vlo[2] = {smem_desc_sw128_lo(smem_u32(&s.v[0][0][0]), kTileBytes),
                                   smem_desc_sw128_lo(smem_u32(&s.v[1][0][0]), kTileBytes)};
          auto issue_qk = [&](int t, int st) {
            const uint32_t a = qlo[t], b = klo[st];
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = ((kk >> 2) * kTileBytes + (kk & 3) * 32) >> 4;  // K-step of 16 columns
              mma_bf16_ss_w(tS[t], a + off, b + off, dhi, id_qk, kk > 0 ? 1u : 0u);
            }
          };
          auto issue_pv = [&](int t, int st, uint32_t acc) {
            const uint32_t b = vlo[st];
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // K-step of 16 keys: 8 TMEM columns of P, 2048 bytes of V
              mma_bf16_ts_w(tO[t], tS[t] + kk * 8, b + kk * (2048 >> 4), dhi, id_pv, (acc || kk > 0) ? 1u : 0u);
          };
          bool ok = mbar_wait(&s.q_full[0], 0, abort_word, p.dc.err) &&
                    mbar_wait(&s.q_full[1], 0, abort_word, p.dc.err) &&
                    mbar_wait(&s.k_full[0], 0, abort_word, p.dc.err);
          if (ok) {
            tc_fence_after_sync();
            issue_qk(0, 0);
            mma_commit(&s.s_full[0]);
            issue_qk(1, 0);
            mma_commit(&s.s_full[1]);
            mma_commit(&s.k_empty[0]);
          }
          for (int j = 0; j < n && ok; ++j) {
            const int st = j & 1;
            const bool more = j + 1 < n;
            const int st1 = (j + 1) & 1;
            const int64_t kb1 = more ? static_cast<int64_t>(ent1 & 0xFFFFFF) * kTile : 0;
            ent1 = j + 2 < n ? ld_keep_s32(list + j + 2) : 0;
            const int c0 = more ? dca_class(R0, kb1, p.dca) : cls[0];
            const int c1 = more ? dca_class(R0 + kTile, kb1, p.dca) : cls[1];
            // V(j) and K(j+1) normally landed long ago: wait for them before P_0(j), so
            // that PV_t(j) and S_t(j + 1) go to the tensor pipe back to back once P_t(j)
            // is stored (the pipe runs dry while this thread does anything else)
            ok = mbar_wait(&s.v_full[st], (j >> 1) & 1, abort_word, p.dc.err) &&
                 (!more || mbar_wait(&s.k_full[st1], ((j + 1) >> 1) & 1, abort_word, p.dc.err));
            // tile 0
            ok = ok && mbar_wait(&s.p_full[0], j & 1, abort_word, p.dc.err);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv(0, st, j > 0);
            if (more) {
              if (c0 != cls[0]) {  // the tile's DCA class changes: wait for Q_0 at the new rotation
                mma_commit(&s.q_empty[0]);
                ok = mbar_wait(&s.q_full[0], qph[0] & 1, abort_word, p.dc.err);
                ++qph[0];
                cls[0] = c0;
                if (!ok) break;
                tc_fence_after_sync();
              }
              issue_qk(0, st1);
              mma_commit(&s.s_full[0]);
            }
            // tile 1
            ok = mbar_wait(&s.p_full[1], j & 1, abort_word, p.dc.err);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv(1, st, j > 0);
            mma_commit(&s.v_empty[st]);
            if (more) {
              if (c1 != cls[1]) {
                mma_commit(&s.q_empty[1]);
                ok = mbar_wait(&s.q_full[1], qph[1] & 1, abort_word, p.dc.err);
                ++qph[1];
                cls[1] = c1;
                if (!ok) break;
                tc_fence_after_sync();
              }
              issue_qk(1, st1);
              mma_commit(&s.s_full[1]);
              mma_commit(&s.k_empty[st1]);
            }
          }
          mma_commit(&s.drain);
          drain_wait_a(&s.drain, 0, p.dc.wait_ns);
        }
        mbar_arrive(&s.o_final);
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const int wl = warp & 3;
    const int m = wl * 32 + lane;
    const int64_t i = R0 + t * kTile + m;  // absolute query position of this row
    const uint32_t tS = tbase + t * 128 + (static_cast<uint32_t>(wl * 32) << 16);
    const uint32_t tO = tbase + 256 + t * 128 + (static_cast<uint32_t>(wl * 32) << 16);
    const uint32_t* vb = p.vbits + static_cast<int64_t>(h) * p.nwords;
    const uint32_t* sb = p.sbits + static_cast<int64_t>(h) * p.nwords;
    float m_run = -INFINITY, l_run = 0.f;
    int32_t ent = n > 0 ? list[0] : 0;  // schedule entry of block j, read a block ahead
    unsigned long long useful = 0;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int32_t entry = ent;
      ent = j + 1 < n ? ld_keep_s32(list + j + 1) : 0;
      const int64_t k0 = static_cast<int64_t>(entry & 0xFFFFFF) * kTile;
      const int state = (entry >> (24 + 2 * t)) & 3;
      // element mask of this row over the block's 128 keys
      uint32_t mw[4];
      if (state == 0 || i >= p.e) {
        mw[0] = mw[1] = mw[2] = mw[3] = 0u;
      } else {
        if (state == 2) {
          mw[0] = mw[1] = mw[2] = mw[3] = 0xFFFFFFFFu;
        } else {
          const uint4 vv = *reinterpret_cast<const uint4*>(vb + (k0 >> 5));
          const int64_t dlo = i - k0 - 127;  // >= -127
          const int64_t wd = (dlo >> 5) + kSPad;
          const int sh = static_cast<int>(dlo & 31);
          uint32_t w5[5];
#pragma unroll
          for (int q = 0; q < 5; ++q) w5[q] = sb[wd + q];
          uint32_t x[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) x[q] = __funnelshift_r(w5[q], w5[q + 1], sh);
          mw[0] = vv.x | __brev(x[3]);
          mw[1] = vv.y | __brev(x[2]);
          mw[2] = vv.z | __brev(x[1]);
          mw[3] = vv.w | __brev(x[0]);
        }
        const int64_t lim = i - k0;  // causal: column c <= i - k0
        if (lim < 127) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t cm;
            if (lim >= 32 * q + 31)
              cm = 0xFFFFFFFFu;
            else if (lim < 32 * q)
              cm = 0u;
            else
              cm = (2u << (lim - 32 * q)) - 1u;
            mw[q] &= cm;
          }
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[t], j & 1, abort_word, p.dc.err));
      if (!ok) break;
      tc_fence_after_sync();
      useful += __popc(mw[0]) + __popc(mw[1]) + __popc(mw[2]) + __popc(mw[3]);
      // Optimistic softmax: a row that already has a reference max is exponentiated
      // against it without a max pass. A block whose row sum exceeds 2^16 (so some p
      // may exceed 2^16) is redone from S, which stays in tensor memory until P is
      // stored, with its true max and the lazy-rescale rule; so is every block of a
      // warp with a row still without reference.
      bool optimistic = __all_sync(0xffffffffu, m_run != -INFINITY);
      uint32_t pk[64];
      float lsum = 0.f;
#pragma unroll 1
      for (int attempt = 0; attempt < 2; ++attempt) {
        // the row's 128 scores: four tcgen05.ld and one wait
        float sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32];
          tmem_ld32(tS + c * 32, raw);
#pragma unroll
          for (int x = 0; x < 32; ++x) sv[c * 32 + x] = __uint_as_float(raw[x]);
        }
        tmem_wait_ld();
        // element mask; blocks where every lane keeps all 128 keys skip the selects
        const bool all_on = __all_sync(0xffffffffu, (mw[0] & mw[1] & mw[2] & mw[3]) == 0xFFFFFFFFu);
        if (!all_on) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) sv[c] = -INFINITY;
        }
        if (!optimistic) {
          // row max of the raw scores: 8 chains of 3-input max (scale > 0 keeps the order)
          float mx[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            mx[x] = fmax3(sv[x], sv[x + 8], sv[x + 16]);
#pragma unroll
            for (int c = 24; c < 120; c += 16) mx[x] = fmax3(mx[x], sv[x + c], sv[x + c + 8]);
            mx[x] = fmaxf(mx[x], sv[x + 120]);
          }
          const float mblk =
              fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
              p.scale_log2;
          // lazy rescale: move the reference max only when it grows by > 2^8
          const float m_new = fmaxf(m_run, mblk);
          const bool need = m_new > m_run + kRescaleThreshold;
          const float f = need ? ex2a(m_run - m_new) : 1.0f;  // 0 when m_run = -inf
          // O_t holds PV_t(j-1) complete: S_t(j) was committed after it
          if (j > 0 && __any_sync(0xffffffffu, need && m_run != -INFINITY)) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * f);
              tmem_st32(tO + c * 32, o);
            }
            tmem_wait_st();
          }
          if (need) {
            l_run *= f;
            m_run = m_new;
          }
        }
        // p = exp2(s * scale * log2(e) - m): the arguments of two columns per packed
        // fp32x2 FMA, one MUFU exp2 per element, the row sum over 4 packed chains, P as
        // bf16 pairs (issue slots, not a pipe, bound this warp's loop)
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t sc2 = f32x2_pack(p.scale_log2, p.scale_log2), nm2 = f32x2_pack(nm, nm);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          float a0, a1;
          f32x2_unpack(f32x2_fma(f32x2_pack(sv[2 * c], sv[2 * c + 1]), sc2, nm2), a0, a1);
          const float p0 = ex2a(a0), p1 = ex2a(a1);
          ls2[c & 3] = f32x2_add(ls2[c & 3], f32x2_pack(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
        lsum = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float u0, u1;
          f32x2_unpack(ls2[x], u0, u1);
          lsum += u0 + u1;
        }
        if (optimistic && __any_sync(0xffffffffu, lsum > kOptimisticSum)) {
          optimistic = false;
          continue;
        }
        break;
      }
      l_run += lsum;
      tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(pk));
      tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full[t]);
    }
    // ---------------------------------------------------------- epilogue
    const bool fin = __all_sync(0xffffffffu, mbar_wait(&s.o_final, 0, abort_word, p.dc.err));
    tc_fence_after_sync();
    if (fin && ok) {
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
      const int64_t orow = i - p.q_pos0;
      uint16_t* dst = p.out + (static_cast<int64_t>(h) * p.out_rows + orow) * kD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        if (i < p.e) {
          uint32_t pkd[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pkd[x] = l_run > 0.f ? pack_bf16x2(__uint_as_float(o[2 * x]) * inv,
                                               __uint_as_float(o[2 * x + 1]) * inv)
                                 : 0u;  // a row without selected keys is written as zeros
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
        }
      }
      if (i < p.e && p.lse_out)
        p.lse_out[static_cast<int64_t>(h) * p.out_rows + orow] =
            l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) useful += __shfl_xor_sync(0xffffffffu, useful, o);
    if (lane == 0 && useful) atomicAdd(p.stats + 1, useful);
  }
  // ------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 512);
  }
}

vs_status run_sparse_prefill(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                             int64_t e, const uint16_t* k, const uint16_t* v, int64_t kv_rows,
                             const int32_t* v_idx, int32_t cap_v, const int32_t* v_cnt,
                             const int32_t* s_off, int32_t cap_s, const int32_t* s_cnt,
                             uint16_t* out, float* lse_out, cudaStream_t st) {
  const Layout& L = c->L;
  const int hq = c->cfg.hq, hkv = c->cfg.hkv, g = hq / hkv;
  const int64_t nrows = e - q_pos0;
  const bool dca = c->dca.enabled != 0;
  vs_status s;
  // rotated keys at DCA key positions (or continuous ones)
  s = ensure_keys_rotated(c, k, kv_rows, e, dca, st);
  if (s != VS_OK) return s;
  // rotated chunk queries, one copy per DCA class
  bf16* qrot = ws_ptr<bf16>(c, L.q_rot);
  for (int var = 0; var < L.nvar; ++var) {
    const int mode = dca ? 2 + var : 0;
    s = launch_rope_rows(c, reinterpret_cast<const bf16*>(q), q_rows, 0,
                         qrot + static_cast<int64_t>(var) * hq * L.rows_pad * kD, L.rows_pad, 0, 1,
                         L.rows_pad, 0, nrows, hq, q_pos0, mode, st);
    if (s != VS_OK) return s;
  }
  // bitmaps of the selected sets, slash prefix counts, per-CTA block lists
  uint32_t* vbits = ws_ptr<uint32_t>(c, L.vbits);
  uint32_t* sbits = ws_ptr<uint32_t>(c, L.sbits);
  uint32_t* scum = ws_ptr<uint32_t>(c, L.scum);
  s = cuda_check(cudaMemsetAsync(vbits, 0, static_cast<size_t>(hq) * L.nwords * 4, st), "bitmap clear");
  if (s == VS_OK) s = cuda_check(cudaMemsetAsync(sbits, 0, static_cast<size_t>(hq) * L.nwords * 4, st), "bitmap clear");
  if (s == VS_OK) s = cuda_check(cudaMemsetAsync(c->stats, 0, 2 * sizeof(unsigned long long), st), "stats clear");
  if (s != VS_OK) return s;
  set_bits_kernel<<<dim3(64, hq, 2), 256, 0, st>>>(v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt, e, vbits,
                                                  sbits, L.nwords, c->err);
  s = launched("set_bits_kernel launch");
  if (s != VS_OK) return s;
  prefix_popc_kernel<<<hq, 1024, 0, st>>>(sbits, L.nwords, scum);
  s = launched("prefix_popc_kernel launch");
  if (s != VS_OK) return s;
  const int npairs = static_cast<int>(ceil_div(nrows, 256));
  schedule_kernel<<<dim3(npairs, hq), 256, 0, st>>>(vbits, sbits, scum, L.nwords, q_pos0, e,
                                                   static_cast<int>(L.npairs), L.nblk,
                                                   ws_ptr<int32_t>(c, L.sched),
                                                   ws_ptr<int32_t>(c, L.sched_cnt), c->stats);
  s = launched("schedule launch");
  if (s != VS_OK) return s;
  // tensor maps
  CUtensorMap tmQ, tmK, tmV;
  s = make_tmap_rows(&tmQ, qrot, static_cast<int64_t>(L.nvar) * hq, nrows, L.rows_pad, kTile);
  if (s == VS_OK)
    s = make_tmap_rows(&tmK, c->ws + (dca ? L.k_dca : L.k_cont), hkv, e, c->max_seq, kTile);
  if (s == VS_OK) s = make_tmap_rows(&tmV, v, hkv, e, kv_rows, kTile);
  if (s != VS_OK) return s;
  AttnParams ap{};
  ap.q_pos0 = q_pos0;
  ap.e = e;
  ap.hq = hq;
  ap.g = g;
  ap.npairs = npairs;
  ap.nvar = L.nvar;
  ap.scale_log2 = c->cfg.softmax_scale * kLog2eA;
  ap.sched = ws_ptr<int32_t>(c, L.sched);
  ap.sched_cnt = ws_ptr<int32_t>(c, L.sched_cnt);
  ap.npairs_ws = static_cast<int>(L.npairs);
  ap.nblk_ws = L.nblk;
  ap.vbits = vbits;
  ap.sbits = sbits;
  ap.nwords = L.nwords;
  ap.out = out;
  ap.out_rows = q_rows;
  ap.lse_out = lse_out;
  ap.stats = c->stats;
  ap.dca = c->dca;
  ap.dc = dev_common(c);
  const size_t smem = sizeof(AttnSmem) + 1024;
  cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (c->ev_start) {
    s = cuda_check(cudaEventRecord(c->ev_start, st), "timing event");
    if (s != VS_OK) return s;
  }
  attn_kernel<<<static_cast<unsigned>(npairs) * hq, kAttnThreads, smem, st>>>(tmQ, tmK, tmV, ap);
  s = launched("attn_kernel launch");
  if (s == VS_OK && c->ev_stop) s = cuda_check(cudaEventRecord(c->ev_stop, st), "timing event");
  return s;
}

// ---------------------------------------------------------------- wait self-test
__global__ void wait_selftest_kernel(DevCommon dc) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the wait must run out and report it
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > dc.wait_ns) {
        ok = false;
        break;
      }
    }
    if (!ok) atomicCAS(dc.err, 0, kDevErrTimeout);
    (void)abort_word;
  }
}

vs_status launch_wait_selftest(vs_ctx* c, uint64_t limit_ns, cudaStream_t st) {
  DevCommon dc{c->err, limit_ns};
  wait_selftest_kernel<<<1, 32, 0, st>>>(dc);
  return launched("wait_selftest_kernel launch");
}

}  // namespace vs
