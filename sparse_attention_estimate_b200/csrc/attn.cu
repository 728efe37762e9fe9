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
// Work lists of at least this many entries (K and V of 1024 key blocks per KV head: 64 MB)
// are swept from where the CTAs of their KV head are loading (see attn_kernel).
constexpr int kSweepMin = 1024;
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

// Selected slash offsets in [lo, hi] (inclusive, clipped to the valid offsets by the caller).
__device__ __forceinline__ uint32_t slash_count(const uint32_t* sb, const uint32_t* sc, int64_t lo, int64_t hi) {
  if (hi < lo) return 0u;
  return bit_prefix(sb, sc, hi + 1 + 32 * kSPad) - bit_prefix(sb, sc, lo + 32 * kSPad);
}

// Entry of a work list: bits 0..23 key block (or gather group) index, bits 24..27 the
// two query tiles' states (0 skip, 1 partial, 2 full), bit 28 a gather group, bit 29 a
// key block holding gathered columns (its mask drops them) or a gather group whose
// columns can follow some of the pair's rows (its mask is causal).
constexpr int32_t kEntGroup = 1 << 28;
constexpr int32_t kEntFlag = 1 << 29;
constexpr int32_t kCntGroups = 1 << 30;  // in a list's count: the list holds gather groups

// Gather plan of one head for the chunk of rows [q_pos0, e): which key blocks' vertical
// columns are gathered into dense 128-column groups instead of executing the blocks.
// A block's verticals cost, per pair of query tiles that can see them, either the whole
// block (unless the block's selected offsets make the pair execute it anyway) or
// count/128 of a gathered tile: they are gathered when that is cheaper summed over the
// pairs. Gathered columns leave the masks of the blocks, so each selected element is
// computed once. Writes gbits (the gathered columns' bitmap), gscan (gathered columns
// before each block), glist (the gathered columns, ascending), and the group table:
// consecutive runs of up to 128 gathered columns that never cross a DCA chunk boundary,
// gkoff[k] the first group of key chunk k (gkoff[nk] the number of groups).
__global__ void __launch_bounds__(1024) gather_plan_kernel(
    const uint32_t* __restrict__ vbits, const uint32_t* __restrict__ sbits,
    const uint32_t* __restrict__ scum, int64_t nwords, int64_t q_pos0, int64_t e, int npairs,
    DcaParams dca, int64_t nblk_ws, int64_t gcap, int64_t nkmax, uint32_t* __restrict__ gbits,
    int32_t* __restrict__ gscan, int32_t* __restrict__ glist, int4* __restrict__ gtab,
    int32_t* __restrict__ gkoff, int64_t e_pad) {
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t* vb = vbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sb = sbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sc = scum + static_cast<int64_t>(h) * (nwords + 1);
  uint32_t* gb = gbits + static_cast<int64_t>(h) * nwords;
  int32_t* gs = gscan + static_cast<int64_t>(h) * (nblk_ws + 1);
  int32_t* gl = glist + static_cast<int64_t>(h) * e_pad;
  int4* gt = gtab + static_cast<int64_t>(h) * gcap;
  int32_t* gk = gkoff + static_cast<int64_t>(h) * (nkmax + 1);
  const int64_t nb = (e + kTile - 1) / kTile;
  // 1. decision and gathered count per block
  for (int64_t b = tid; b < nb; b += blockDim.x) {
    const uint4 v = *reinterpret_cast<const uint4*>(vb + 4 * b);
    const int c = __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    bool g = false;
    if (c > 0 && c < kTile) {
      // pairs with a row at or after the block's first key: R0 + 255 >= 128 b
      const int64_t need = kTile * b - 255 - q_pos0;
      const int64_t p_min = need <= 0 ? 0 : (need + 255) / 256;
      const int64_t n_vis = npairs - p_min;
      if (n_vis > 0) {
        const int64_t limit = n_vis * (kTile - c);  // gather iff 128 * cover < limit
        int64_t cover = 0;
        for (int64_t p = p_min; p < npairs && kTile * cover < limit; ++p) {
          const int64_t R0 = q_pos0 + 256 * p;
          const int64_t lo = max(R0 - kTile * b - 127, static_cast<int64_t>(0));
          const int64_t hi = min(min(R0 + 255, e - 1) - kTile * b, e - 1);
          if (slash_count(sb, sc, lo, hi) > 0u) ++cover;
        }
        g = kTile * cover < limit;
      }
    }
    *reinterpret_cast<uint4*>(gb + 4 * b) = g ? v : make_uint4(0u, 0u, 0u, 0u);
    gs[b] = g ? c : 0;
  }
  __syncthreads();
  // 2. exclusive scan of the counts over the blocks (gs[nb] = total)
  __shared__ int wsum[32];
  int running = 0;
  for (int64_t b0 = 0; b0 < nb; b0 += blockDim.x) {
    const int64_t b = b0 + tid;
    const int v = b < nb ? gs[b] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      wsum[lane] = t;
    }
    __syncthreads();
    if (b < nb) gs[b] = running + (w > 0 ? wsum[w - 1] : 0) + x - v;
    running += wsum[31];
    __syncthreads();
  }
  if (tid == 0) gs[nb] = running;
  __syncthreads();
  // 3. the gathered columns, ascending
  for (int64_t b = tid; b < nb; b += blockDim.x) {
    const uint4 v = *reinterpret_cast<const uint4*>(gb + 4 * b);
    const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
    int pos = gs[b];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t m = ws[q];
      while (m) {
        const int x = __ffs(m) - 1;
        m &= m - 1u;
        gl[pos++] = static_cast<int32_t>(kTile * b + 32 * q + x);
      }
    }
  }
  // 4. groups: per DCA key chunk k (blocks [k S/128, (k+1) S/128)), runs of 128 columns
  const int64_t sblk = dca.enabled ? dca.S / kTile : nb;  // blocks per key chunk (S % 128 == 0)
  const int64_t nk = (nb + sblk - 1) / sblk;
  if (tid == 0) {
    int32_t g = 0;
    for (int64_t k = 0; k < nk; ++k) {
      gk[k] = g;
      const int64_t c0 = gs[k * sblk], c1 = gs[min((k + 1) * sblk, nb)];
      g += static_cast<int32_t>((c1 - c0 + kTile - 1) / kTile);
    }
    gk[nk] = g;
  }
  __syncthreads();
  const int32_t ng = gk[nk];
  for (int32_t g = tid; g < ng; g += blockDim.x) {
    int64_t lo = 0, hi = nk - 1;  // the key chunk k with gk[k] <= g < gk[k + 1]
    while (lo < hi) {
      const int64_t mid = (lo + hi + 1) / 2;
      if (gk[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int64_t k = lo;
    const int64_t c0 = gs[k * sblk], c1 = gs[min((k + 1) * sblk, nb)];
    const int64_t start = c0 + static_cast<int64_t>(g - gk[k]) * kTile;
    const int cnt = static_cast<int>(min(static_cast<int64_t>(kTile), c1 - start));
    gt[g] = make_int4(static_cast<int>(start), cnt, static_cast<int>(k), gl[start]);
  }
}

// State of (query tile starting at R0, key block starting at k0): 0 skip, 1 partial, 2 full.
// Gathered columns (gb) do not count: they are computed in their groups. *has_g tells
// whether the block holds gathered columns (its mask must then drop them).
__device__ __forceinline__ int tile_block_state(int64_t R0, int64_t k0, int64_t e,
                                                const uint32_t* vb, const uint32_t* sb,
                                                const uint32_t* sc, const uint32_t* gb,
                                                bool* has_g) {
  const uint4 gv = *reinterpret_cast<const uint4*>(gb + (k0 >> 5));
  *has_g = (gv.x | gv.y | gv.z | gv.w) != 0u;
  if (R0 >= e || k0 > R0 + 127) return 0;
  const int64_t dhi_raw = R0 + 127 - k0;
  const int64_t dlo = R0 - k0 - 127 > 0 ? R0 - k0 - 127 : 0;
  const int64_t dhi = dhi_raw < e - 1 ? dhi_raw : e - 1;
  const uint32_t scount = slash_count(sb, sc, dlo, dhi);
  const bool s_all = dhi >= dlo && scount == static_cast<uint32_t>(dhi - dlo + 1);
  const uint4 v = *reinterpret_cast<const uint4*>(vb + (k0 >> 5));
  const uint32_t vw[4] = {v.x & ~gv.x, v.y & ~gv.y, v.z & ~gv.z, v.w & ~gv.w};
  const bool v_all = (vw[0] & vw[1] & vw[2] & vw[3]) == 0xFFFFFFFFu;
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
  if (v_all || (s_all && !*has_g)) return 2;
  return (v_any || scount > 0) ? 1 : 0;
}

// Work list of one (pair of query tiles, head), key chunk by DCA key chunk (one chunk
// without DCA): the gather groups of the chunk whose first column some row of the pair
// can see, then the chunk's key blocks with a selected non-gathered element for either
// tile. Ordered this way, the DCA class of consecutive entries changes at most twice.
__global__ void __launch_bounds__(256) schedule_kernel(
    const uint32_t* __restrict__ vbits, const uint32_t* __restrict__ sbits,
    const uint32_t* __restrict__ scum, const uint32_t* __restrict__ gbits,
    const int4* __restrict__ gtab, const int32_t* __restrict__ gkoff,
    const int32_t* __restrict__ glist, int64_t e_pad, int64_t nwords, int64_t q_pos0, int64_t e,
    DcaParams dca, int64_t gcap, int64_t nkmax, int npairs_ws, int64_t nsched,
    int32_t* __restrict__ sched, int32_t* __restrict__ sched_cnt, unsigned long long* stats) {
  const int pair = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint32_t* vb = vbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sb = sbits + static_cast<int64_t>(h) * nwords;
  const uint32_t* sc = scum + static_cast<int64_t>(h) * (nwords + 1);
  const uint32_t* gb = gbits + static_cast<int64_t>(h) * nwords;
  const int4* gt = gtab + static_cast<int64_t>(h) * gcap;
  const int32_t* gk = gkoff + static_cast<int64_t>(h) * (nkmax + 1);
  const int64_t R0 = q_pos0 + static_cast<int64_t>(pair) * 256;
  const int64_t last_row = (e - 1 < R0 + 255) ? e - 1 : R0 + 255;
  const int64_t nb = last_row / kTile + 1;
  const int64_t sblk = dca.enabled ? dca.S / kTile : nb;
  const int64_t nk = (nb + sblk - 1) / sblk;
  const int64_t nk_all = ((e + kTile - 1) / kTile + sblk - 1) / sblk;  // key chunks of the plan
  int32_t* out = sched + (static_cast<int64_t>(h) * npairs_ws + pair) * 2 * nsched;
  auto gl_last = [&](int hh, const int4& d) {  // last column of a group
    return static_cast<int64_t>(glist[static_cast<int64_t>(hh) * e_pad + d.x + d.y - 1]);
  };
  __shared__ int wsum[8];
  int running = 0, groups = 0;
  // block-wide compaction of one batch of 256 candidate entries (flagged when non-zero)
  auto emit = [&](bool f, int32_t entry) {
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[w] = __popc(bal);
    __syncthreads();
    int base = running;
    for (int i = 0; i < w; ++i) base += wsum[i];
    int total = 0;
    for (int i = 0; i < 8; ++i) total += wsum[i];
    if (f) out[base + __popc(bal & ((1u << lane) - 1u))] = entry;
    running += total;
    __syncthreads();
  };
  for (int64_t k = 0; k < nk; ++k) {
    // gather groups of key chunk k
    const int32_t g0 = k < nk_all ? gk[k] : 0, g1 = k < nk_all ? gk[k + 1] : 0;
    for (int32_t gb0 = g0; gb0 < g1; gb0 += 256) {
      const int32_t g = gb0 + tid;
      bool f = false;
      int32_t entry = 0;
      const int before = running;
      if (g < g1) {
        const int4 d = gt[g];  // start, count, key chunk, first column
        const int64_t first_col = d.w;
        const int64_t last_col = gl_last(h, d);
        f = first_col <= last_row;
        int flags = 0;
        for (int t = 0; t < 2; ++t) {
          const int64_t r0 = R0 + t * kTile;
          if (r0 >= e || first_col > min(r0 + 127, e - 1)) continue;  // no row of the tile sees it
          // full: 128 columns, all before the tile's first row
          flags |= (d.y == kTile && last_col < r0 ? 2 : 1) << (2 * t);
        }
        // causal mask needed when a column of the group can follow one of the pair's rows
        entry = g | kEntGroup | (flags << 24) | (last_col >= R0 ? kEntFlag : 0);
      }
      emit(f, entry);
      groups += running - before;
    }
    // key blocks of key chunk k
    const int64_t b_lo = k * sblk, b_hi = min((k + 1) * sblk, nb);
    for (int64_t b0 = b_lo; b0 < b_hi; b0 += 256) {
      const int64_t b = b0 + tid;
      int flags = 0;
      bool hg0 = false, hg1 = false;
      if (b < b_hi) {
        const int64_t k0 = b * kTile;
        flags = tile_block_state(R0, k0, e, vb, sb, sc, gb, &hg0) |
                (tile_block_state(R0 + 128, k0, e, vb, sb, sc, gb, &hg1) << 2);
      }
      emit(flags != 0, static_cast<int32_t>(b) | (flags << 24) | (hg0 ? kEntFlag : 0));
    }
  }
  // A list long enough to be swept from another start is written twice in a row, so that
  // the attention CTA reads entries start .. start + n - 1 with no wrap-around.
  if (running >= kSweepMin) {
    __syncthreads();
    for (int i = tid; i < running; i += blockDim.x) out[running + i] = out[i];
  }
  if (tid == 0) {
    // the list's length, and bit 30 when it holds gather groups
    sched_cnt[static_cast<int64_t>(h) * npairs_ws + pair] = running | (groups > 0 ? kCntGroups : 0);
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
  int64_t nsched;
  const uint32_t* vbits;
  const uint32_t* sbits;
  int64_t nwords;
  // gathered vertical columns: bitmap and prefix counts [hq][nwords], the columns
  // [hq][e_pad] and the groups [hq][gcap] (start, count, DCA key chunk, first column)
  const uint32_t* gbits;
  const uint32_t* gcum;
  const int32_t* glist;
  const int4* gtab;
  int64_t e_pad, gcap;
  int dca_sblk;  // key blocks per DCA chunk (S / 128), 0 without DCA
  int* sweep;    // per KV head: list position last loaded by one of its CTAs (a hint)
  int rotate;    // lists of kSweepMin entries or more start at that position
  // row sources of the gathered groups: rotated keys and values, [hkv][rows][128]
  const uint16_t* k_rot;
  int64_t k_rows;
  const uint16_t* v;
  int64_t v_rows;
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
  int gather_ok;  // a stage wait's outcome, shared among the gather threads
  int start;      // first list entry of this CTA's sweep
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

// DCA class of (query tile in DCA chunk qc, keys of DCA chunk kc): 0 intra,
// 1 successive, 2 inter (always 0 without DCA, where every chunk index is 0).
__device__ __forceinline__ int dca_class(int qc, int kc) {
  return qc == kc ? 0 : (qc == kc + 1 ? 1 : 2);
}

// DCA chunk of a work-list entry's keys: a key block's (the chunk stride is sblk
// blocks), or a gather group's (groups never straddle a chunk). 32-bit arithmetic:
// the issuing threads run this for every entry.
__device__ __forceinline__ int entry_kchunk(int32_t ent, const int4* gtab, int64_t gcap, int h, int sblk) {
  if (sblk == 0) return 0;  // no DCA
  const uint32_t idx = static_cast<uint32_t>(ent) & 0xFFFFFFu;
  if (ent & kEntGroup) return gtab[static_cast<int64_t>(h) * gcap + idx].z;
  return static_cast<int>(idx / static_cast<uint32_t>(sblk));
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
  const int32_t* list = p.sched + (static_cast<int64_t>(h) * p.npairs_ws + pair) * 2 * p.nsched;
  // DCA chunks of the two query tiles (fixed for the CTA)
  const int qc0 = p.dca.enabled ? static_cast<int>(R0 / p.dca.S) : 0;
  const int qc1 = p.dca.enabled ? static_cast<int>((R0 + kTile) / p.dca.S) : 0;
  const int cnt_raw = p.sched_cnt[static_cast<int64_t>(h) * p.npairs_ws + pair];
  const int n = cnt_raw & (kCntGroups - 1);
  const bool has_groups = (cnt_raw & kCntGroups) != 0;
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
    // Sweep start: where a CTA of the same KV head loaded last. Once a KV head's keys and
    // values outgrow L2, CTAs that all sweep from block 0 drift apart (SMs run at slightly
    // different speeds, and each takes the next CTA when its own ends) until the blocks a
    // CTA reads have left L2 before the next one reaches them. Joining the CTAs in flight
    // keeps them within a few hundred blocks of each other. The position is kept per KV
    // head: all its query heads read the same blocks (one position per query head let the
    // heads settle at different places, each group reading the blocks on its own). A list
    // of n entries is stored twice in a row, so the sweep start .. start + n - 1 needs no
    // wrap-around; the order of the entries changes only the summation order of the
    // online softmax.
    int start = 0;
    if (p.rotate && n >= kSweepMin)
      start = static_cast<int>(static_cast<uint32_t>(__ldcg(p.sweep + hk)) % static_cast<uint32_t>(n));
    s.start = start;
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
        const int start = s.start;
        const int32_t* lst = list + start;
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int cls[2];
        int qchg[2] = {0, 0};
        const int kc0 = entry_kchunk(lst[0], p.gtab, p.gcap, h, p.dca_sblk);
        for (int t = 0; t < 2; ++t) {
          cls[t] = dca_class(t ? qc1 : qc0, kc0);
          mbar_arrive_expect_tx(&s.q_full[t], 2 * kTileBytes);
          const int qrow = pair * 256 + t * kTile;
          const int qh = cls[t] * p.hq + h;
          tma_load_3d(s.q[t][0], &tmQ, &s.q_full[t], 0, qrow, qh);
          tma_load_3d(s.q[t][1], &tmQ, &s.q_full[t], 64, qrow, qh);
        }
        // per stage: entries seen so far (TMA or gather, each completes one phase of the
        // stage's full barriers) and the phase of the last TMA load issued (-1: none), for
        // draining the copies in flight when the CTA aborts
        int nst[2] = {0, 0}, kph[2] = {-1, -1}, vph[2] = {-1, -1};
        bool ok = true;
        int32_t ent = lst[0];  // schedule entries are read one block ahead of use
        for (int j = 0; j < n && ok; ++j) {
          const int32_t cur = ent;
          const int b = cur & 0xFFFFFF;
          const bool grp = (cur & kEntGroup) != 0;  // a gather group: warps 2-3 load its K and V
          ent = j + 1 < n ? ld_keep_s32(lst + j + 1) : 0;
          const int st = j & 1;
          // K(j) first: the MMA warp releases a Q tile only after issuing S0(j).
          // Both loaders (this one and the gather warps) wait for every entry's stage to
          // empty, their own entries or not: a parity wait is exact only for the phase
          // right after the last one waited for.
          if (j >= 2) ok = mbar_wait(&s.k_empty[st], ((j >> 1) - 1) & 1, abort_word, p.dc.err, 1, j);
          if (!ok) break;
          if (!grp) {
            mbar_arrive_expect_tx(&s.k_full[st], 2 * kTileBytes);
            tma_load_3d(s.k[st][0], &tmK, &s.k_full[st], 0, b * kTile, hk);
            tma_load_3d(s.k[st][1], &tmK, &s.k_full[st], 64, b * kTile, hk);
            kph[st] = nst[st];
          }
          if (p.rotate && n >= kSweepMin && (j & 63) == 0) {  // where this CTA is now
            const int pos = start + j;
            __stcg(p.sweep + hk, pos >= n ? pos - n : pos);
          }
          if (j > 0) {
            const int kc = entry_kchunk(cur, p.gtab, p.gcap, h, p.dca_sblk);
            for (int t = 0; t < 2 && ok; ++t) {
              const int c = dca_class(t ? qc1 : qc0, kc);
              if (c != cls[t]) {
                ok = mbar_wait(&s.q_empty[t], qchg[t] & 1, abort_word, p.dc.err, 2 + t, j);
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
          if (j >= 2) ok = mbar_wait(&s.v_empty[st], ((j >> 1) - 1) & 1, abort_word, p.dc.err, 4, j);
          if (!ok || grp) {
            ++nst[st];
            if (!ok) break;
            continue;
          }
          mbar_arrive_expect_tx(&s.v_full[st], 2 * kTileBytes);
          tma_load_3d(s.v[st][0], &tmV, &s.v_full[st], 0, b * kTile, hk);
          tma_load_3d(s.v[st][1], &tmV, &s.v_full[st], 64, b * kTile, hk);
          vph[st] = nst[st];
          ++nst[st];
        }
        if (!ok) {  // let every issued copy land before the CTA exits
          // A stage's TMA load is issued only after every earlier phase of its barrier has
          // completed, so the phase of the last one is the barrier's current phase.
          for (int t = 0; t < 2; ++t) drain_wait_a(&s.q_full[t], qchg[t] & 1, p.dc.wait_ns);
          for (int st = 0; st < 2; ++st) {
            if (kph[st] >= 0) drain_wait_a(&s.k_full[st], kph[st] & 1, p.dc.wait_ns);
            if (vph[st] >= 0) drain_wait_a(&s.v_full[st], vph[st] & 1, p.dc.wait_ns);
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
          const int32_t* lst = list + s.start;
          const int kc0 = entry_kchunk(lst[0], p.gtab, p.gcap, h, p.dca_sblk);
          cls[0] = dca_class(qc0, kc0);
          cls[1] = dca_class(qc1, kc0);
          int32_t ent1 = n > 1 ? lst[1] : 0;  // entry of block j + 1, read a block ahead
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
          bool ok = mbar_wait(&s.q_full[0], 0, abort_word, p.dc.err, 16, 0) &&
                    mbar_wait(&s.q_full[1], 0, abort_word, p.dc.err, 17, 0) &&
                    mbar_wait(&s.k_full[0], 0, abort_word, p.dc.err, 18, 0);
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
            const int kc1 = more ? entry_kchunk(ent1, p.gtab, p.gcap, h, p.dca_sblk) : 0;
            ent1 = j + 2 < n ? ld_keep_s32(lst + j + 2) : 0;
            const int c0 = more ? dca_class(qc0, kc1) : cls[0];
            const int c1 = more ? dca_class(qc1, kc1) : cls[1];
            // V(j) and K(j+1) normally landed long ago: wait for them before P_0(j), so
            // that PV_t(j) and S_t(j + 1) go to the tensor pipe back to back once P_t(j)
            // is stored (the pipe runs dry while this thread does anything else)
            ok = mbar_wait(&s.v_full[st], (j >> 1) & 1, abort_word, p.dc.err, 5, j) &&
                 (!more || mbar_wait(&s.k_full[st1], ((j + 1) >> 1) & 1, abort_word, p.dc.err, 6, j));
            // tile 0
            ok = ok && mbar_wait(&s.p_full[0], j & 1, abort_word, p.dc.err, 7, j);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv(0, st, j > 0);
            if (more) {
              if (c0 != cls[0]) {  // the tile's DCA class changes: wait for Q_0 at the new rotation
                mma_commit(&s.q_empty[0]);
                ok = mbar_wait(&s.q_full[0], qph[0] & 1, abort_word, p.dc.err, 8, j);
                ++qph[0];
                cls[0] = c0;
                if (!ok) break;
                tc_fence_after_sync();
              }
              issue_qk(0, st1);
              mma_commit(&s.s_full[0]);
            }
            // tile 1
            ok = mbar_wait(&s.p_full[1], j & 1, abort_word, p.dc.err, 9, j);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv(1, st, j > 0);
            mma_commit(&s.v_empty[st]);
            if (more) {
              if (c1 != cls[1]) {
                mma_commit(&s.q_empty[1]);
                ok = mbar_wait(&s.q_full[1], qph[1] & 1, abort_word, p.dc.err, 10, j);
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
    } else {
      // ------------------------------------------------------------ gather loader (warps 2-3)
      // For each gather group of the list: the 128 gathered columns' rotated K rows and
      // V rows, copied 16 bytes at a time into the stage's tiles in the 128-byte-swizzled
      // layout the TMA loads produce (rows past the group's count repeat its first
      // column; their scores are masked). Thread g copies tile rows g and g + 64.
      const int gtid = tid - 64;
      const int32_t* gl = p.glist + static_cast<int64_t>(h) * p.e_pad;
      const int32_t* lst = list + s.start;
      int32_t ent = n > 0 ? lst[0] : 0;
      bool ok = has_groups;  // lists without groups are the TMA producer's alone
      // Every entry's stage-empty phases are waited for (by thread 0, the outcome shared
      // through the named barrier), as in the TMA producer: a parity wait is exact only
      // for the phase right after the last one waited for.
      for (int j = 0; j < n && ok; ++j) {
        const int32_t cur = ent;
        ent = j + 1 < n ? ld_keep_s32(lst + j + 1) : 0;
        const bool grp = (cur & kEntGroup) != 0;
        const int st = j & 1;
        int64_t col[2] = {0, 0};
        if (grp) {
          const int4 d = p.gtab[static_cast<int64_t>(h) * p.gcap + (cur & 0xFFFFFF)];  // start, count, key chunk, first column
          col[0] = gl[d.x + (gtid < d.y ? gtid : 0)];
          col[1] = gl[d.x + (gtid + 64 < d.y ? gtid + 64 : 0)];
        }
        for (int kvh = 0; kvh < 2 && ok; ++kvh) {  // K rows into k[st], then V rows into v[st]
          if (j >= 2) {
            if (gtid == 0)
              s.gather_ok = mbar_wait(kvh == 0 ? &s.k_empty[st] : &s.v_empty[st], ((j >> 1) - 1) & 1, abort_word,
                                      p.dc.err, 11 + kvh, j)
                                ? 1
                                : 0;
            named_barrier_sync(1, 64);
            ok = s.gather_ok != 0;
            named_barrier_sync(1, 64);  // every thread has read the outcome before the next wait
          }
          if (!ok) break;  // uniform over the 64 threads: nothing was copied
          if (!grp) continue;
          const uint16_t* base = kvh == 0 ? p.k_rot : p.v;
          const int64_t rows = kvh == 0 ? p.k_rows : p.v_rows;
          bf16 (*dst)[kTile * 64] = kvh == 0 ? s.k[st] : s.v[st];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int r = gtid + 64 * rr;
            const uint16_t* src = base + (static_cast<int64_t>(hk) * rows + col[rr]) * kD;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              char* d8 = reinterpret_cast<char*>(&dst[c >> 3][0]) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
              cp_async_16(d8, src + c * 8);
            }
          }
          cp_async_wait_all();
          fence_proxy_async_smem();  // the MMA reads these tiles through the async proxy
          named_barrier_sync(1, 64);
          if (gtid == 0) mbar_arrive(kvh == 0 ? &s.k_full[st] : &s.v_full[st]);
        }
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
    const int32_t* lst = list + s.start;
    int32_t ent = n > 0 ? lst[0] : 0;  // schedule entry of block j, read a block ahead
    unsigned long long useful = 0;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int32_t entry = ent;
      ent = j + 1 < n ? ld_keep_s32(lst + j + 1) : 0;
      const int64_t k0 = static_cast<int64_t>(entry & 0xFFFFFF) * kTile;
      const int state = (entry >> (24 + 2 * t)) & 3;
      // element mask of this row over the block's (or gather group's) 128 keys
      uint32_t mw[4];
      if (state == 0 || i >= p.e) {
        mw[0] = mw[1] = mw[2] = mw[3] = 0u;
      } else if (entry & kEntGroup) {
        // gather group: its first `count` columns, those at or before this row when the
        // group reaches into the pair's rows (columns ascending: a prefix of the group)
        const int4 d = p.gtab[static_cast<int64_t>(h) * p.gcap + (entry & 0xFFFFFF)];
        int nvalid = d.y;
        if (entry & kEntFlag) {
          const int64_t wi = static_cast<int64_t>(h) * p.nwords + (i >> 5);
          const int64_t upto = static_cast<int64_t>(p.gcum[wi + h]) +  // gcum rows hold nwords + 1 entries
                               __popc(p.gbits[wi] & ((2u << static_cast<int>(i & 31)) - 1u));  // gathered columns <= i
          const int64_t nv = upto - d.x;
          nvalid = nv < 0 ? 0 : (nv > d.y ? d.y : static_cast<int>(nv));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          mw[q] = nvalid >= 32 * (q + 1) ? 0xFFFFFFFFu : (nvalid > 32 * q ? (1u << (nvalid - 32 * q)) - 1u : 0u);
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
          if (entry & kEntFlag) {  // gathered columns are computed in their groups
            const uint4 gv = *reinterpret_cast<const uint4*>(p.gbits + static_cast<int64_t>(h) * p.nwords + (k0 >> 5));
            mw[0] &= ~gv.x;
            mw[1] &= ~gv.y;
            mw[2] &= ~gv.z;
            mw[3] &= ~gv.w;
          }
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
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[t], j & 1, abort_word, p.dc.err, 13 + t, j));
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
    const bool fin = __all_sync(0xffffffffu, mbar_wait(&s.o_final, 0, abort_word, p.dc.err, 15, 0));
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
  // vertical columns gathered into dense groups where that beats executing their blocks
  uint32_t* gbits = ws_ptr<uint32_t>(c, L.gbits);
  uint32_t* gcum = ws_ptr<uint32_t>(c, L.gcum);
  s = cuda_check(cudaMemsetAsync(gbits, 0, static_cast<size_t>(hq) * L.nwords * 4, st), "gather bitmap clear");
  if (s != VS_OK) return s;
  gather_plan_kernel<<<hq, 1024, 0, st>>>(vbits, sbits, scum, L.nwords, q_pos0, e, npairs, c->dca, L.nblk,
                                          L.gcap, L.nkmax, gbits, ws_ptr<int32_t>(c, L.gscan),
                                          ws_ptr<int32_t>(c, L.glist), ws_ptr<int4>(c, L.gtab),
                                          ws_ptr<int32_t>(c, L.gkoff), L.e_pad);
  s = launched("gather_plan_kernel launch");
  if (s != VS_OK) return s;
  prefix_popc_kernel<<<hq, 1024, 0, st>>>(gbits, L.nwords, gcum);
  s = launched("prefix_popc_kernel launch");
  if (s != VS_OK) return s;
  schedule_kernel<<<dim3(npairs, hq), 256, 0, st>>>(
      vbits, sbits, scum, gbits, ws_ptr<int4>(c, L.gtab), ws_ptr<int32_t>(c, L.gkoff),
      ws_ptr<int32_t>(c, L.glist), L.e_pad, L.nwords, q_pos0, e, c->dca, L.gcap, L.nkmax,
      static_cast<int>(L.npairs), L.nsched, ws_ptr<int32_t>(c, L.sched), ws_ptr<int32_t>(c, L.sched_cnt),
      c->stats);
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
  ap.sweep = ws_ptr<int>(c, L.sweep);
  ap.rotate = c->deterministic ? 0 : 1;
  ap.nsched = L.nsched;
  ap.vbits = vbits;
  ap.sbits = sbits;
  ap.nwords = L.nwords;
  ap.gbits = gbits;
  ap.gcum = gcum;
  ap.glist = ws_ptr<int32_t>(c, L.glist);
  ap.gtab = ws_ptr<int4>(c, L.gtab);
  ap.e_pad = L.e_pad;
  ap.gcap = L.gcap;
  ap.dca_sblk = dca ? static_cast<int>(c->dca.S / kTile) : 0;
  ap.k_rot = reinterpret_cast<const uint16_t*>(c->ws + (dca ? L.k_dca : L.k_cont));
  ap.k_rows = c->max_seq;
  ap.v = v;
  ap.v_rows = kv_rows;
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
