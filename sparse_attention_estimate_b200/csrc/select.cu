// select.cu - top-k selection of vertical columns and slash offsets, and the
// refinement decision.
//
// The vertical-slash step of the Qwen2.5-1M explainer ("Sparse Attention",
// step 3) keeps, per head, the k_v columns with the largest vertical score and
// the k_s diagonal offsets with the largest slash score; "Sparsity Refinement"
// doubles both budgets while the head's attention recall is below the
// threshold. Every budget of a refinement run is a level t with
// k_t = min(k_base * 2^t, e); since the ranking (score descending, index
// ascending) is fixed, the selected sets are nested and one pass can assign each
// column / offset the first level that selects it.
//
// Every (head, array) is cut into segments, one CTA each (several per array, so
// that the arrays of all heads fill the SMs); threads load 16 bytes at a time.
//  radix select   the k_t-th largest key of every level at once, four 8-bit digit
//                 passes over the fp32 bit pattern (which orders non-negative
//                 floats): per pass a histogram kernel over the segments and a
//                 decide kernel per (head, array) that fixes the digit; the state
//                 between passes (prefixes, ranks, distinct prefixes) lives in the
//                 workspace. The result: the threshold key of each level and how
//                 many elements equal to it are taken (lowest index first).
//  levels         each element's first level (255: none); the order of elements
//                 equal to a threshold (by index) comes from per-segment counts.
//  compact        the ascending index list of one level per head, segments placed
//                 by their counts.
//  refine_decide  first level whose recall reaches tau (or saturation).
#include <algorithm>

#include "internal.cuh"

namespace vs {

constexpr uint32_t kNoThreshold = 0xFFFFFFFFu;  // level with k = 0: selects nothing
constexpr int kDevErrCap = 3;                    // an output list was longer than its cap
constexpr int kSelThreads = 512;                 // threads of the segment kernels
constexpr int kSelTile = 4 * kSelThreads;        // elements per tile: four per thread

// Sort key of element j: fp32 bit pattern of a non-negative score (0 for
// non-positive or NaN), +inf for slash offset 0, which is always selected.
__device__ __forceinline__ uint32_t sel_key(float x, int64_t j, int arr) {
  if (arr == 1 && j == 0) return 0x7F800000u;
  return (x > 0.0f) ? __float_as_uint(x) : 0u;
}

// The four keys of elements j0 .. j0+3 of array x (keys of elements at or past `hi`
// are 0, and such elements are reported invalid by the callers). vec: x is 16-byte
// aligned at every multiple of 4.
__device__ __forceinline__ void load_keys4(const float* x, int64_t j0, int64_t hi, int arr, bool vec,
                                           uint32_t (&k)[4]) {
  if (vec && j0 + 3 < hi) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(x + j0));
    k[0] = sel_key(v.x, j0, arr);
    k[1] = sel_key(v.y, j0 + 1, arr);
    k[2] = sel_key(v.z, j0 + 2, arr);
    k[3] = sel_key(v.w, j0 + 3, arr);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) k[q] = j0 + q < hi ? sel_key(__ldg(x + j0 + q), j0 + q, arr) : 0u;
  }
}

// Exclusive block-wide prefix sum of v over the CTA's threads (blockDim.x ==
// kSelThreads); *total gets the sum. wsum: 32 ints of shared memory.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const int base = (w > 0) ? wsum[w - 1] : 0;
  *total = wsum[nw - 1];
  __syncthreads();
  return base + x - v;
}

// Radix-select state of one (head, array) between passes.
struct RadixState {
  uint32_t prefix[kMaxLevels];   // digits of the level's threshold fixed so far
  uint32_t uprefix[kMaxLevels];  // distinct prefixes of the active levels
  int32_t slot[kMaxLevels];      // the level's entry in uprefix (-1: inactive level)
  int32_t nu;                    // distinct prefixes
  int32_t pad;
  long long rank[kMaxLevels];    // rank still to find among the elements with the prefix
};

__device__ __forceinline__ const float* sel_row(const float* vert, const float* slash, int64_t e_ld, int h,
                                                int arr) {
  return (arr == 0 ? vert : slash) + static_cast<int64_t>(h) * e_ld;
}

// Level budgets k_t = min(base * 2^t, e) (base <= 0: the level selects nothing); all
// active levels start with the empty prefix.
__global__ void radix_init_kernel(const int32_t* __restrict__ kv, const int32_t* __restrict__ ks, int64_t e,
                                  int nlev, RadixState* __restrict__ rs) {
  const int h = blockIdx.y, arr = blockIdx.x, t = threadIdx.x;
  RadixState& st = rs[h * 2 + arr];
  __shared__ int any;
  if (t == 0) any = 0;
  __syncthreads();
  if (t < kMaxLevels) {
    int64_t base = (arr == 0) ? kv[h] : ks[h];
    if (base < 0) base = 0;
    int64_t k = 0;
    if (t < nlev && base > 0) {
      k = (t < 40 && base <= (e >> t)) ? (base << t) : e;
      if (k > e) k = e;
    }
    st.prefix[t] = 0;
    st.rank[t] = k;
    st.slot[t] = k > 0 ? 0 : -1;
    if (k > 0) atomicOr(&any, 1);
  }
  __syncthreads();
  if (t == 0) {
    st.uprefix[0] = 0;
    st.nu = any ? 1 : 0;
  }
}

// One digit pass: histograms of digit (key >> shift) & 255 of the segment's elements,
// per distinct prefix (the key's bits above the digit), into part[(h,arr,seg)][slot][256].
__global__ void __launch_bounds__(kSelThreads) radix_hist_kernel(
    const float* __restrict__ vert, const float* __restrict__ slash, int64_t e_ld, int64_t e, int64_t seg,
    bool vec, int shift, const RadixState* __restrict__ rs, uint32_t* __restrict__ part, int nslot) {
  const int b = blockIdx.x, arr = blockIdx.y, h = blockIdx.z, tid = threadIdx.x;
  const RadixState& st = rs[h * 2 + arr];
  const int nu = st.nu;
  if (nu == 0) return;
  extern __shared__ uint32_t hist[];  // [nu][256]
  __shared__ uint32_t sp[kMaxLevels];  // the distinct prefixes, ascending
  __shared__ int su[kMaxLevels];       // their slots in the state
  for (int i = tid; i < nu * 256; i += blockDim.x) hist[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < nu; ++i) {  // insertion sort of at most kMaxLevels prefixes
      const uint32_t v = st.uprefix[i];
      int j = i;
      for (; j > 0 && sp[j - 1] > v; --j) {
        sp[j] = sp[j - 1];
        su[j] = su[j - 1];
      }
      sp[j] = v;
      su[j] = i;
    }
  }
  __syncthreads();
  const float* x = sel_row(vert, slash, e_ld, h, arr);
  const int64_t lo = static_cast<int64_t>(b) * seg, hi = min(lo + seg, e);
  for (int64_t t0 = lo; t0 < hi; t0 += kSelTile) {  // the same trip count for every thread
    const int64_t j0 = t0 + 4 * tid;
    uint32_t k[4];
    load_keys4(x, j0, hi, arr, vec, k);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int u = -1;
      uint32_t digit = 0;
      if (j0 + q < hi) {
        const uint32_t hp = shift == 24 ? 0u : (k[q] >> (shift + 8));
        int l0 = 0, l1 = nu;  // bisection: first sorted prefix >= hp
        while (l0 < l1) {
          const int mid = (l0 + l1) >> 1;
          if (sp[mid] < hp)
            l0 = mid + 1;
          else
            l1 = mid;
        }
        if (l0 < nu && sp[l0] == hp) u = su[l0];
        digit = (k[q] >> shift) & 255u;
      }
      if (shift == 24) {
        // first digit (sign and high exponent bits): scores of one array share a few
        // values, so equal digits of the warp add once
        const uint32_t tag = u < 0 ? 0xFFFFFFFFu : digit;
        const uint32_t peers = __match_any_sync(0xffffffffu, tag);
        if (u >= 0 && (__ffs(peers) - 1) == (tid & 31)) atomicAdd(&hist[digit], __popc(peers));
      } else if (u >= 0) {
        // lower digits spread over the bins: a plain shared-memory add per key
        atomicAdd(&hist[u * 256 + digit], 1u);
      }
    }
  }
  __syncthreads();
  uint32_t* o = part + (static_cast<int64_t>(h * 2 + arr) * gridDim.x + b) * nslot * 256;
  for (int i = tid; i < nu * 256; i += blockDim.x) o[i] = hist[i];
}

// Fixes one digit of every active level from the segments' histograms; after the last
// pass (final) writes the thresholds thr[(h,arr)][t] = (key, how many equal keys to take).
__global__ void __launch_bounds__(256) radix_decide_kernel(RadixState* __restrict__ rs,
                                                           const uint32_t* __restrict__ part, int nseg,
                                                           int nslot, bool final, int nlev,
                                                           uint32_t* __restrict__ thr) {
  const int arr = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  RadixState& st = rs[h * 2 + arr];
  const int nu = st.nu;
  __shared__ uint32_t hist[kMaxLevels][256];
  const uint32_t* pp = part + static_cast<int64_t>(h * 2 + arr) * nseg * nslot * 256;
  for (int u = 0; u < nu; ++u) {
    uint32_t sum = 0;
    for (int b = 0; b < nseg; ++b) sum += pp[(static_cast<int64_t>(b) * nslot + u) * 256 + tid];
    hist[u][tid] = sum;
  }
  __syncthreads();
  if (tid < kMaxLevels && st.slot[tid] >= 0) {
    const int u = st.slot[tid];
    long long cum = 0;
    const long long r = st.rank[tid];
    for (int d = 255; d >= 0; --d) {
      const long long cnt = hist[u][d];
      if (cum + cnt >= r) {
        st.prefix[tid] = (st.prefix[tid] << 8) | static_cast<uint32_t>(d);
        st.rank[tid] = r - cum;
        break;
      }
      cum += cnt;
    }
  }
  __syncthreads();
  if (tid == 0) {  // distinct prefixes of the active levels, for the next pass
    int n = 0;
    for (int t = 0; t < kMaxLevels; ++t) {
      if (st.slot[t] < 0) continue;
      int u = 0;
      while (u < n && st.uprefix[u] != st.prefix[t]) ++u;
      if (u == n) st.uprefix[n++] = st.prefix[t];
      st.slot[t] = u;
    }
    st.nu = n;
  }
  __syncthreads();
  if (final && tid < kMaxLevels) {
    uint32_t* o = thr + (static_cast<int64_t>(h) * 2 + arr) * kMaxLevels * 2 + 2 * tid;
    const bool ok = tid < nlev && st.slot[tid] >= 0;
    o[0] = ok ? st.prefix[tid] : kNoThreshold;
    o[1] = ok ? static_cast<uint32_t>(st.rank[tid]) : 0u;
  }
}

// The distinct threshold keys of one (head, array) into shared memory; returns how many.
__device__ __forceinline__ int load_thresholds(const uint32_t* thr, int h, int arr, int nlev, uint32_t* T,
                                               uint32_t* take, uint32_t* uT) {
  __shared__ int nu_s;
  if (threadIdx.x == 0) {
    int nu = 0;
    for (int t = 0; t < nlev; ++t) {
      const uint32_t* p = thr + ((static_cast<int64_t>(h) * 2 + arr) * kMaxLevels + t) * 2;
      T[t] = p[0];
      take[t] = p[1];
      if (p[0] == kNoThreshold) continue;
      int u = 0;
      while (u < nu && uT[u] != p[0]) ++u;
      if (u == nu) uT[nu++] = p[0];
    }
    for (int i = 1; i < nu; ++i) {  // ascending, for the bisection of find_threshold
      const uint32_t v = uT[i];
      int j = i;
      for (; j > 0 && uT[j - 1] > v; --j) uT[j] = uT[j - 1];
      uT[j] = v;
    }
    nu_s = nu;
  }
  __syncthreads();
  return nu_s;
}

// Index of key k among the nu distinct threshold keys uT (ascending), -1 if none.
__device__ __forceinline__ int find_threshold(const uint32_t* uT, int nu, uint32_t k) {
  int l0 = 0, l1 = nu;
  while (l0 < l1) {
    const int mid = (l0 + l1) >> 1;
    if (uT[mid] < k)
      l0 = mid + 1;
    else
      l1 = mid;
  }
  return (l0 < nu && uT[l0] == k) ? l0 : -1;
}

// Per segment: how many elements equal each distinct threshold key, into
// cnt[(h,arr,seg)][u].
__global__ void __launch_bounds__(kSelThreads) eq_count_kernel(
    const float* __restrict__ vert, const float* __restrict__ slash, int64_t e_ld, int64_t e, int64_t seg,
    bool vec, int nlev, const uint32_t* __restrict__ thr, int32_t* __restrict__ cnt) {
  const int b = blockIdx.x, arr = blockIdx.y, h = blockIdx.z, tid = threadIdx.x;
  __shared__ uint32_t T[kMaxLevels], take[kMaxLevels], uT[kMaxLevels];
  __shared__ int c_s[kMaxLevels];
  if (tid < kMaxLevels) c_s[tid] = 0;
  const int nu = load_thresholds(thr, h, arr, nlev, T, take, uT);
  const float* x = sel_row(vert, slash, e_ld, h, arr);
  const int64_t lo = static_cast<int64_t>(b) * seg, hi = min(lo + seg, e);
  for (int64_t t0 = lo; t0 < hi; t0 += kSelTile) {
    const int64_t j0 = t0 + 4 * tid;
    uint32_t k[4];
    load_keys4(x, j0, hi, arr, vec, k);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (j0 + q < hi) {
        const int u = find_threshold(uT, nu, k[q]);
        if (u >= 0) atomicAdd(&c_s[u], 1);
      }
  }
  __syncthreads();
  if (tid < kMaxLevels) cnt[(static_cast<int64_t>(h * 2 + arr) * gridDim.x + b) * kMaxLevels + tid] = c_s[tid];
}

// Each element's first level: key above the level's threshold, or equal to it and among
// the first `take` such elements by index (255: no level selects it).
__global__ void __launch_bounds__(kSelThreads) levels_kernel(
    const float* __restrict__ vert, const float* __restrict__ slash, int64_t e_ld, int64_t e, int64_t seg,
    bool vec, int nlev, const uint32_t* __restrict__ thr, const int32_t* __restrict__ cnt,
    uint8_t* __restrict__ lvl, int64_t e_pad) {
  const int b = blockIdx.x, arr = blockIdx.y, h = blockIdx.z, tid = threadIdx.x;
  __shared__ uint32_t T[kMaxLevels], take[kMaxLevels], uT[kMaxLevels];
  __shared__ long long run[kMaxLevels];
  __shared__ int wsum[32];
  const int nu = load_thresholds(thr, h, arr, nlev, T, take, uT);
  if (tid < nu) {  // equal keys in the earlier segments
    long long r = 0;
    for (int bb = 0; bb < b; ++bb) r += cnt[(static_cast<int64_t>(h * 2 + arr) * gridDim.x + bb) * kMaxLevels + tid];
    run[tid] = r;
  }
  __syncthreads();
  const float* x = sel_row(vert, slash, e_ld, h, arr);
  uint8_t* out = lvl + (static_cast<int64_t>(h) * 2 + arr) * e_pad;
  const int64_t lo = static_cast<int64_t>(b) * seg, hi = min(lo + seg, e);
  for (int64_t t0 = lo; t0 < hi; t0 += kSelTile) {
    const int64_t j0 = t0 + 4 * tid;
    uint32_t k[4];
    load_keys4(x, j0, hi, arr, vec, k);
    int myu[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) myu[q] = j0 + q < hi ? find_threshold(uT, nu, k[q]) : -1;
    long long rk[4] = {0, 0, 0, 0};
    const bool mine = myu[0] >= 0 || myu[1] >= 0 || myu[2] >= 0 || myu[3] >= 0;
    if (__syncthreads_or(mine)) {
      for (int u = 0; u < nu; ++u) {
        const int c = (myu[0] == u) + (myu[1] == u) + (myu[2] == u) + (myu[3] == u);
        if (!__syncthreads_or(c > 0)) continue;
        int total = 0;
        int r = block_excl_scan(c, wsum, &total);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (myu[q] == u) rk[q] = run[u] + r++;
        __syncthreads();
        if (tid == 0) run[u] += total;
        __syncthreads();
      }
    }
    uint32_t packed = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t level = 255;
      if (j0 + q < hi) {
        // The thresholds do not increase with the level (the budgets grow), so the
        // levels whose threshold is at most the key are a suffix: find its start t0 by
        // bisection. Levels with no threshold (kNoThreshold) precede the others.
        int lo_t = 0, hi_t = nlev;  // first t with T[t] <= key (T[t] != kNoThreshold)
        while (lo_t < hi_t) {
          const int mid = (lo_t + hi_t) >> 1;
          const uint32_t tt = T[mid];
          if (tt != kNoThreshold && tt <= k[q])
            hi_t = mid;
          else
            lo_t = mid + 1;
        }
        // from t0 on: a key above the threshold is selected; a key equal to it is
        // selected among the first take[t] equal keys (the next levels take more)
        for (int t = lo_t; t < nlev; ++t) {
          const uint32_t tt = T[t];
          if (k[q] > tt || rk[q] < static_cast<long long>(take[t])) {
            level = static_cast<uint32_t>(t);
            break;
          }
        }
      }
      packed |= level << (8 * q);
    }
    if (j0 + 3 < hi)
      *reinterpret_cast<uint32_t*>(out + j0) = packed;  // j0 % 4 == 0, rows 128-aligned
    else
      for (int q = 0; q < 4; ++q)
        if (j0 + q < hi) out[j0 + q] = static_cast<uint8_t>(packed >> (8 * q));
  }
}

// The four level bytes of elements j0 .. j0+3 that are at or below level tsel.
__device__ __forceinline__ int selected4(const uint8_t* lv, int64_t j0, int64_t hi, int tsel, bool (&f)[4]) {
  uint32_t w4 = 0xFFFFFFFFu;
  if (j0 + 3 < hi)
    w4 = *reinterpret_cast<const uint32_t*>(lv + j0);
  else
    for (int q = 0; q < 4; ++q)
      if (j0 + q < hi) w4 = (w4 & ~(0xFFu << (8 * q))) | (static_cast<uint32_t>(lv[j0 + q]) << (8 * q));
  int c = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[q] = static_cast<int>((w4 >> (8 * q)) & 0xFFu) <= tsel;
    c += f[q];
  }
  return c;
}

// Per segment: elements selected at the head's chosen level (level 0 without a choice).
__global__ void __launch_bounds__(kSelThreads) compact_count_kernel(const uint8_t* __restrict__ lvl,
                                                                    int64_t e_pad, int64_t e, int64_t seg,
                                                                    const int32_t* __restrict__ choice,
                                                                    int32_t* __restrict__ cnt) {
  const int b = blockIdx.x, arr = blockIdx.y, h = blockIdx.z, tid = threadIdx.x;
  const uint8_t* lv = lvl + (static_cast<int64_t>(h) * 2 + arr) * e_pad;
  const int tsel = choice ? choice[h] : 0;
  const int64_t lo = static_cast<int64_t>(b) * seg, hi = min(lo + seg, e);
  int c = 0;
  for (int64_t t0 = lo; t0 < hi; t0 += kSelTile) {
    bool f[4];
    c += selected4(lv, t0 + 4 * tid, hi, tsel, f);
  }
  __shared__ int wsum[32];
  int total = 0;
  block_excl_scan(c, wsum, &total);
  if (tid == 0) cnt[static_cast<int64_t>(h * 2 + arr) * gridDim.x + b] = total;
}

// The ascending index list of the selected elements: the segment's elements go after
// those of the earlier segments. The last segment's CTA writes the list length.
__global__ void __launch_bounds__(kSelThreads) compact_write_kernel(
    const uint8_t* __restrict__ lvl, int64_t e_pad, int64_t e, int64_t seg, const int32_t* __restrict__ choice,
    const int32_t* __restrict__ cnt, int32_t* v_idx, int32_t cap_v, int32_t* v_cnt, int32_t* s_off,
    int32_t cap_s, int32_t* s_cnt, int* err) {
  const int b = blockIdx.x, arr = blockIdx.y, h = blockIdx.z, tid = threadIdx.x;
  const uint8_t* lv = lvl + (static_cast<int64_t>(h) * 2 + arr) * e_pad;
  const int tsel = choice ? choice[h] : 0;
  const int32_t cap = arr == 0 ? cap_v : cap_s;
  int32_t* out = arr == 0 ? v_idx + static_cast<int64_t>(h) * cap_v : s_off + static_cast<int64_t>(h) * cap_s;
  const int32_t* cc = cnt + static_cast<int64_t>(h * 2 + arr) * gridDim.x;
  __shared__ int wsum[32];
  __shared__ long long base_s;
  if (tid == 0) {
    long long r = 0;
    for (int bb = 0; bb < b; ++bb) r += cc[bb];
    base_s = r;
  }
  __syncthreads();
  long long running = base_s;
  const int64_t lo = static_cast<int64_t>(b) * seg, hi = min(lo + seg, e);
  for (int64_t t0 = lo; t0 < hi; t0 += kSelTile) {
    const int64_t j0 = t0 + 4 * tid;
    bool f[4];
    const int c = selected4(lv, j0, hi, tsel, f);
    int total = 0;
    long long pos = running + block_excl_scan(c, wsum, &total);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (f[q]) {
        if (pos < cap) out[pos] = static_cast<int32_t>(j0 + q);
        ++pos;
      }
    running += total;
  }
  if (b == static_cast<int>(gridDim.x) - 1 && tid == 0) {
    (arr == 0 ? v_cnt : s_cnt)[h] = static_cast<int32_t>(running < cap ? running : cap);
    if (running > cap) atomicCAS(err, 0, kDevErrCap);
  }
}

__global__ void refine_decide_kernel(const float* __restrict__ hist, int nsplit, int hq, int nlev,
                                     int nr, int64_t e, float tau, int32_t* kv, int32_t* ks,
                                     float* recall, int32_t* choice, const float* __restrict__ base_rc,
                                     const int* __restrict__ base_dec) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= hq) return;
  int64_t kv0 = kv[h] < 0 ? 0 : kv[h], ks0 = ks[h] < 0 ? 0 : ks[h];
  if (base_dec && base_dec[h]) {  // the base budgets reach tau (their recall from the sums)
    choice[h] = 0;
    kv[h] = static_cast<int32_t>(kv0 > e ? e : kv0);
    ks[h] = static_cast<int32_t>(ks0 > e ? e : ks0);
    recall[h] = base_rc[h];
    return;
  }
  double cum = 0.0;
  int chosen = nlev - 1;
  int64_t kvt = 0, kst = 0;
  double rc = 0.0;
  for (int t = 0; t < nlev; ++t) {
    double m = 0.0;
    for (int s = 0; s < nsplit; ++s)
      m += static_cast<double>(hist[(static_cast<int64_t>(s) * hq + h) * kMaxLevels + t]);
    cum = m;  // the histogram is cumulative: level t holds the recall mass of C_t
    rc = cum / nr;
    kvt = (kv0 << t) > e ? e : (kv0 << t);
    kst = (ks0 << t) > e ? e : (ks0 << t);
    if (t > 0 && (kv0 << (t - 1)) >= e) kvt = e;
    if (t > 0 && (ks0 << (t - 1)) >= e) kst = e;
    if (rc >= static_cast<double>(tau) || (kvt >= e && kst >= e) || t == nlev - 1) {
      chosen = t;
      break;
    }
  }
  choice[h] = chosen;
  kv[h] = static_cast<int32_t>(kvt);
  ks[h] = static_cast<int32_t>(kst);
  recall[h] = static_cast<float>(rc);
}

// Offline calibration: acc[h] = max(acc[h], budget[h]) for both budgets.
__global__ void budgets_max_kernel(int hq, const int32_t* __restrict__ kv, const int32_t* __restrict__ ks,
                                   int32_t* kv_acc, int32_t* ks_acc) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= hq) return;
  kv_acc[h] = max(kv_acc[h], kv[h]);
  ks_acc[h] = max(ks_acc[h], ks[h]);
}

vs_status run_budgets_max(int hq, const int32_t* kv, const int32_t* ks, int32_t* kv_acc, int32_t* ks_acc,
                          cudaStream_t st) {
  budgets_max_kernel<<<static_cast<unsigned>(ceil_div(hq, 128)), 128, 0, st>>>(hq, kv, ks, kv_acc, ks_acc);
  return launched("budgets_max_kernel launch");
}

vs_status run_refine_decide(vs_ctx* c, int64_t e, int nr, int nlev, float tau, int32_t* kv,
                            int32_t* ks, float* recall, bool base_decided, cudaStream_t st) {
  refine_decide_kernel<<<static_cast<unsigned>(ceil_div(c->cfg.hq, 64)), 64, 0, st>>>(
      ws_ptr<float>(c, c->L.hist), c->hist_nsplit, c->cfg.hq, nlev, nr, e, tau, kv, ks, recall,
      ws_ptr<int32_t>(c, c->L.choice), base_decided ? ws_ptr<float>(c, c->L.base_rc) : nullptr,
      base_decided ? ws_ptr<int>(c, c->L.base_rc) + c->cfg.hq : nullptr);
  return launched("refine_decide_kernel launch");
}


// Segments per (head, array): enough CTAs over all heads to fill the SMs about four
// times, each segment at least one tile and a multiple of the tile.
int select_max_segments(int hq);
int select_segments(int hq, int64_t e, int64_t* seg_out) {
  int nseg = select_max_segments(hq);
  nseg = static_cast<int>(std::min<int64_t>(nseg, ceil_div(e, kSelTile)));
  nseg = std::max(1, nseg);
  const int64_t seg = round_up(ceil_div(e, nseg), kSelTile);
  *seg_out = seg;
  return static_cast<int>(ceil_div(e, seg));
}

vs_status launch_select(const SelScratch& sc, int hq, const float* vert, const float* slash, int64_t e_ld,
                        int64_t e, const int32_t* kv, const int32_t* ks, int nlev, const int32_t* choice,
                        int32_t* v_idx, int32_t cap_v, int32_t* v_cnt, int32_t* s_off, int32_t cap_s,
                        int32_t* s_cnt, bool thresholds_and_levels, bool compact, cudaStream_t st) {
  int64_t seg = 0;
  const int nseg = select_segments(hq, e, &seg);
  const bool vec = (e_ld % 4) == 0 && (reinterpret_cast<uintptr_t>(vert) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(slash) & 15u) == 0;
  const dim3 grid(nseg, 2, hq);
  vs_status s = VS_OK;
  if (thresholds_and_levels) {
    RadixState* rs = reinterpret_cast<RadixState*>(sc.state);
    radix_init_kernel<<<dim3(2, hq), 32, 0, st>>>(kv, ks, e, nlev, rs);
    s = launched("radix_init_kernel launch");
    for (int pass = 0; pass < 4 && s == VS_OK; ++pass) {
      radix_hist_kernel<<<grid, kSelThreads, nlev * 256 * sizeof(uint32_t), st>>>(
          vert, slash, e_ld, e, seg, vec, 24 - 8 * pass, rs, sc.part, nlev);
      s = launched("radix_hist_kernel launch");
      if (s != VS_OK) break;
      radix_decide_kernel<<<dim3(2, hq), 256, 0, st>>>(rs, sc.part, nseg, nlev, pass == 3, nlev, sc.thr);
      s = launched("radix_decide_kernel launch");
    }
    if (s != VS_OK) return s;
    int32_t* cnt = reinterpret_cast<int32_t*>(sc.part);  // the histograms are consumed
    eq_count_kernel<<<grid, kSelThreads, 0, st>>>(vert, slash, e_ld, e, seg, vec, nlev, sc.thr, cnt);
    s = launched("eq_count_kernel launch");
    if (s != VS_OK) return s;
    levels_kernel<<<grid, kSelThreads, 0, st>>>(vert, slash, e_ld, e, seg, vec, nlev, sc.thr, cnt, sc.lvl,
                                                sc.e_pad);
    s = launched("levels_kernel launch");
    if (s != VS_OK) return s;
  }
  if (compact) {
    int32_t* cnt = reinterpret_cast<int32_t*>(sc.part);
    compact_count_kernel<<<grid, kSelThreads, 0, st>>>(sc.lvl, sc.e_pad, e, seg, choice, cnt);
    s = launched("compact_count_kernel launch");
    if (s != VS_OK) return s;
    compact_write_kernel<<<grid, kSelThreads, 0, st>>>(sc.lvl, sc.e_pad, e, seg, choice, cnt, v_idx, cap_v,
                                                       v_cnt, s_off, cap_s, s_cnt, sc.err);
    s = launched("compact_write_kernel launch");
  }
  return s;
}

int select_max_segments(int hq) {
  return std::max(1, std::min(static_cast<int>(ceil_div(4 * 148, 2 * hq)), kSelMaxSegments));
}
size_t sel_state_bytes(int hq) { return static_cast<size_t>(hq) * 2 * sizeof(RadixState); }
size_t sel_part_bytes(int hq, int nslot) {
  return static_cast<size_t>(hq) * 2 * select_max_segments(hq) * nslot * 256 * sizeof(uint32_t);
}

}  // namespace vs
