// Multi-level mask generation: query-block means, block logits against the
// level-3 pooled keys, per-query-block softmax, ranking and threshold cuts.
//
// Method: top168.com article on PSA (arXiv:2512.04025), component two (levels
// are allocated from the importance of query-key block pairs) and the ablation
// paragraph (threshold-based allocation beats quantile-based); abstract of
// "PSA: Pyramid Sparse Attention for Efficient Video Understanding and
// Generation" (lower pooling levels for critical KV blocks, higher ones for
// the rest).  How a query block is summarised, how the 8 level-3 keys of a KV
// block become one logit, and how masses become levels are readings of this
// implementation: q_bar = mean of the valid rows; z_j = logsumexp_g(s q_bar.K3_g
// + ln c_g); P = softmax_j(z); rank by P descending (ties to the lower j); a
// block ranked r takes the smallest level l with C_r < tau_l, C_r the mass of
// the blocks ranked before it, else it is pruned.
//
// Three launches (the block logits themselves are in score_tc.cu):
//   qmean_kernel   one CTA per query block; streams Q once (HBM-bound).
//   score_tc_kernel  split-precision tensor-core GEMM of query-block means
//                  against the level-3 keys, logsumexp per KV block fused.
//   assign_kernel  one warp per query block: softmax, a candidate cut (the
//                  blocks above a bisected mass threshold, a prefix of the
//                  ranking) sorted in registers, or a bitonic sort of the whole
//                  row's packed (P, index) keys; scan, levels, overrides, and
//                  the work list (KV block indices grouped by level).
#include "psa_internal.cuh"

namespace psa {
namespace {

// -------------------------------------------------------------- q means

// One CTA of q_blk * d / 64 threads per query block (256 for 128 x 128, 128
// for 128 x 64 or 64 x 128): thread t takes the 8-column chunk t % (d/8) of
// rows t / (d/8) + k * parts (parts = threads / (d/8), k < 8), so that every
// thread issues 8 loads, all before adding.  Lanes holding the same chunk are
// summed with shuffles, the warps' partial sums in shared memory.
template <typename T> struct QVec;
template <> struct QVec<__nv_bfloat16> {
  uint4 raw;
  __device__ void load(const __nv_bfloat16* p) { raw = *reinterpret_cast<const uint4*>(p); }
  __device__ void add_to(float* acc) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __bfloat1622float2(h[i]);
      acc[2 * i] += v.x;
      acc[2 * i + 1] += v.y;
    }
  }
};
template <> struct QVec<float> {
  float4 u, w;
  __device__ void load(const float* p) {
    u = reinterpret_cast<const float4*>(p)[0];
    w = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ void add_to(float* acc) const {
    acc[0] += u.x; acc[1] += u.y; acc[2] += u.z; acc[3] += u.w;
    acc[4] += w.x; acc[5] += w.y; acc[6] += w.z; acc[7] += w.w;
  }
};

template <typename T>
__global__ void __launch_bounds__(256) qmean_kernel(MaskArgs a, const T* __restrict__ Q,
                                                    float* __restrict__ qmh,
                                                    float* __restrict__ qml) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;               // (b*Hq + h) * Nq + qa
  const int qa = row % a.Nq;
  const long long bh = row / a.Nq;
  const int lo = qa * a.q_blk;
  const int n = min(a.q_blk, a.N - lo);
  const int chunks = a.d / 8;               // 16 or 8
  const int parts = blockDim.x / chunks;    // rows read side by side
  const int c = threadIdx.x % chunks;
  const int part = threadIdx.x / chunks;
  const T* base = Q + (bh * a.N + lo) * a.d + c * 8;
  QVec<T> raw[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = part + k * parts;
    if (r < n) raw[k].load(base + (long long)r * a.d);
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (part + k * parts < n) raw[k].add_to(acc);
  // lanes l, l + chunks, ... of a warp hold the same chunk
  for (int o = chunks; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  __shared__ float red[8][16][8];           // [warp][chunk][column]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  if (lane < chunks)
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane][e] = acc[e];
  __syncthreads();
  if (threadIdx.x < chunks) {
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = red[0][c][e];
    for (int w = 1; w < nwarps; ++w)
#pragma unroll
      for (int e = 0; e < 8; ++e) sum[e] += red[w][c][e];
    // the mean in fp32, stored as tf32 head + exact tail
    float hd[8], tl[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float m = __fdiv_rn(sum[e], (float)n);
      hd[e] = tf32_head(m);
      tl[e] = m - hd[e];
    }
    float4* dh = reinterpret_cast<float4*>(qmh + (long long)row * a.d + c * 8);
    float4* dl = reinterpret_cast<float4*>(qml + (long long)row * a.d + c * 8);
    dh[0] = make_float4(hd[0], hd[1], hd[2], hd[3]);
    dh[1] = make_float4(hd[4], hd[5], hd[6], hd[7]);
    dl[0] = make_float4(tl[0], tl[1], tl[2], tl[3]);
    dl[1] = make_float4(tl[4], tl[5], tl[6], tl[7]);
  }
}

// -------------------------------------------------------------- scoring

// ------------------------------------------------------------ assignment
//
// One warp per query block: no block-wide barriers.  The warp keeps its row's
// packed (P, index) keys in shared memory and sorts them with a bitonic
// network (lanes take strided compare-exchanges, __syncwarp between stages).

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <typename T>
__device__ __forceinline__ T warp_excl_scan(T v, T* total) {
  const int lane = threadIdx.x & 31;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// Writes the work list of one query block from its level row `lev` (shared,
// padded with -1 up to a multiple of 16 bytes): KV block indices at level 0,
// then 1, 2, 3, each in increasing index order.  Each lane owns a contiguous,
// 16-byte aligned run of the row, read 16 levels at a time; byte-wise SIMD
// compares count and locate each level, and two packed scans (two 16-bit
// counts per word; a row has at most 8192 blocks) give every lane its
// positions.
__device__ void emit_list_warp(const int8_t* lev, int Nk, int* __restrict__ list_row,
                               int4* __restrict__ count_row) {
  const int lane = threadIdx.x & 31;
  const int per = (((Nk + 31) / 32) + 15) & ~15;
  const int j0 = lane * per, j1 = min(Nk, j0 + per);
  int cnt[kLevels] = {0, 0, 0, 0};
  for (int j = j0; j < j1; j += 16) {
    const uint4 w = *reinterpret_cast<const uint4*>(lev + j);
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int l = 0; l < kLevels; ++l) cnt[l] += __popc(__vcmpeq4(x[k], 0x01010101u * l)) >> 3;
  }
  int t01, t23;
  const int p01 = warp_excl_scan(cnt[0] | (cnt[1] << 16), &t01);
  const int p23 = warp_excl_scan(cnt[2] | (cnt[3] << 16), &t23);
  const int tot[kLevels] = {t01 & 0xffff, t01 >> 16, t23 & 0xffff, t23 >> 16};
  int pos[kLevels];
  pos[0] = p01 & 0xffff;
  pos[1] = tot[0] + (p01 >> 16);
  pos[2] = tot[0] + tot[1] + (p23 & 0xffff);
  pos[3] = tot[0] + tot[1] + tot[2] + (p23 >> 16);
  for (int j = j0; j < j1; j += 16) {
    const uint4 w = *reinterpret_cast<const uint4*>(lev + j);
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int l = 0; l < kLevels; ++l) {
        uint32_t m = __vcmpeq4(x[k], 0x01010101u * l);   // 0xff in every matching byte
        while (m) {
          const int b = __ffs(m) - 1;                     // lowest bit of the lowest match
          list_row[pos[l]++] = j + 4 * k + (b >> 3);
          m &= ~(0xffu << (b & ~7));
        }
      }
    }
  }
  if (lane == 0) *count_row = make_int4(tot[0], tot[1], tot[2], tot[3]);
}

// Bitonic sort of 32*K 64-bit keys held in registers, descending.  Element
// i = lane*K + r lives in register r of lane `lane`; partners at distance < K
// are in the same lane, others are exchanged with shuffles.
template <int K>
__device__ __forceinline__ void warp_bitonic_desc(unsigned long long (&v)[K]) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int k = 2; k <= 32 * K; k <<= 1) {
    // stages whose partner is in another lane (distance >= K)
#pragma unroll 1
    for (int sd = k >> 1; sd >= K; sd >>= 1) {
      const int lx = sd / K;                // partner lane = lane ^ lx
      const bool upper = (lane & lx) != 0;  // this lane holds the larger index
#pragma unroll
      for (int r = 0; r < K; ++r) {
        const bool desc = ((lane * K + r) & k) == 0;
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[r], lx);
        const bool keep_max = desc != upper;  // descending pairs keep the max at the lower index
        v[r] = keep_max ? (v[r] > o ? v[r] : o) : (v[r] < o ? v[r] : o);
      }
    }
    // stages inside a lane (distance < K), unrolled so registers stay static
#pragma unroll
    for (int sd = K / 2; sd > 0; sd >>= 1) {
      if (sd < k) {
#pragma unroll
        for (int r = 0; r < K; ++r) {
          const int rp = r ^ sd;
          if (rp > r) {
            const bool desc = ((lane * K + r) & k) == 0;
            const unsigned long long x = v[r], y = v[rp];
            const bool swap = desc ? (x < y) : (x > y);
            v[r] = swap ? y : x;
            v[rp] = swap ? x : y;
          }
        }
      }
    }
  }
}

// Candidate set of the register path: at most kCand blocks, kCandPerLane
// keys per lane.
constexpr int kCandPerLane = 4;
constexpr int kCand = 32 * kCandPerLane;

// Rows of more than 1024 blocks keep their keys in shared memory; their
// candidate set holds up to kCandS blocks, kCandPerLaneS per lane.
constexpr int kCandPerLaneS = 8;
constexpr int kCandS = 32 * kCandPerLaneS;

// Shared-memory bytes of one row's keys.  K > 0: the register path (a
// candidate set past kCandPerLane keys per lane).  K = 0: all n2 keys (for
// the bitonic sort of the whole row) and a candidate set.  K < 0, the compact
// path of long rows: the visible blocks' P as floats and a candidate set.
__host__ __device__ inline size_t assign_key_bytes(int K, int n2, int Nk) {
  if (K < 0) return (size_t)((Nk + 31) & ~31) * 4 + (size_t)kCandS * 8;
  return K == 0 ? (size_t)(n2 + kCandS) * 8 : (K > kCandPerLane ? (size_t)kCand * 8 : 0);
}

// The level of a visible block from its place in the ranking.  Threshold
// rule: the smallest l whose tau_l is above c, the mass of the blocks ranked
// before it.  Quantile rule: the smallest l with rank < K_l, where K_l =
// ceil(tau_l * n_visible) is computed exactly in double (a float times an
// integer below 2^14 is exact there).
struct LevelRule {
  bool quantile;
  float tau[kLevels];
  int quota[kLevels];
  __device__ LevelRule(const MaskArgs& a, int nvis) {
    quantile = a.assign == PSA_ASSIGN_QUANTILE;
#pragma unroll
    for (int l = 0; l < kLevels; ++l) {
      tau[l] = a.tau[l];
      quota[l] = (int)ceil((double)a.tau[l] * (double)nvis);
    }
  }
  __device__ __forceinline__ int8_t level(float c, int rank) const {
    int l = -1;
#pragma unroll
    for (int t = kLevels - 1; t >= 0; --t)
      if (quantile ? rank < quota[t] : c < tau[t]) l = t;
    return (int8_t)l;
  }
};

// Sorted keys (descending; lane L holds ranks L*K .. L*K + K - 1) -> levels of
// the first n ranks, with the exclusive running mass c of each.
template <int K>
__device__ __forceinline__ void levels_from_sorted(const unsigned long long (&v)[K], int n,
                                                   const LevelRule& rule, int8_t* lev) {
  const int lane = threadIdx.x & 31;
  float mine = 0.f;
#pragma unroll
  for (int r = 0; r < K; ++r)
    if (lane * K + r < n) mine += __uint_as_float((unsigned)(v[r] >> 32));
  float total;
  float c = warp_excl_scan(mine, &total);
#pragma unroll
  for (int r = 0; r < K; ++r) {
    if (lane * K + r < n) {
      const int j = (int)(0xffffffffu - (unsigned)(v[r] & 0xffffffffu));
      lev[j] = rule.level(c, lane * K + r);
      c += __uint_as_float((unsigned)(v[r] >> 32));
    }
  }
}

template <int K>
__global__ void assign_kernel(MaskArgs a, int n2, int rows_per_cta, int nrows,
                              const float* __restrict__ zlog, const int8_t* __restrict__ maxlev,
                              int8_t* __restrict__ map_ws,
                              int8_t* __restrict__ map_user, float* __restrict__ mass_user,
                              int* __restrict__ list, int4* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * rows_per_cta + warp;
  if (row >= nrows) return;                 // whole warp; no block barriers below
  const int lev_stride = (a.Nk + 15) & ~15;
  // keys in shared memory: all n2 of them for the shared-memory sort, the
  // candidate set for the register path
  const size_t key_bytes = assign_key_bytes(K, n2, a.Nk);
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem) + (size_t)warp * (key_bytes / 8);
  int8_t* lev = reinterpret_cast<int8_t*>(smem + (size_t)rows_per_cta * key_bytes) +
                (size_t)warp * lev_stride;

  const int qa = row % a.Nq;
  const int q_lo = qa * a.q_blk;
  const int q_hi = min(a.N, q_lo + a.q_blk) - 1;
  const int nvis = a.causal ? min(a.Nk, q_hi / a.kv_blk + 1) : a.Nk;
  const float* z = zlog + (long long)row * a.Nk;
  const LevelRule rule(a, nvis);

  // softmax over the visible blocks
  float mx = -INFINITY;
  for (int j = lane; j < nvis; j += 32) mx = fmaxf(mx, z[j]);
  mx = warp_max(mx);
  float part = 0.f;
  for (int j = lane; j < nvis; j += 32) part += expf(z[j] - mx);
  const float inv = 1.0f / warp_sum(part);
  auto make_key = [&](int i) -> unsigned long long {
    if (i >= nvis) return 0ull;
    const float pj = expf(z[i] - mx) * inv;
    return ((unsigned long long)__float_as_uint(pj) << 32) | (0xffffffffu - (unsigned)i);
  };
  for (int j = lane; j < lev_stride; j += 32) lev[j] = -1;

  // rank by P descending (ties to the lower index); the level from the
  // exclusive running mass (threshold rule) or the rank (quantile rule)
  if constexpr (K > 0) {
    // P of element i = lane*K + r in register r (0 past the visible blocks)
    float pj[K];
#pragma unroll
    for (int r = 0; r < K; ++r) {
      const int i = lane * K + r;
      pj[r] = i < nvis ? expf(z[i] - mx) * inv : 0.f;
    }
    __syncwarp();                          // lev[] initialised by all lanes
    bool done = false;
    if constexpr (K > kCandPerLane) {
      // Candidate cut: blocks with P >= t form a prefix of the ranking.
      // Threshold rule: when their mass reaches tau_3 every block after them
      // has a running mass >= tau_3, i.e. is pruned (a margin of 1e-3 on the
      // mass keeps the rounding of this sum against the running masses below
      // from mattering).  Quantile rule: when they number at least K_3, every
      // block after them has rank >= K_3.  t is bisected until the candidates
      // number at most kCand; then only the candidates are ranked.
      const float target = a.tau[kLevels - 1] + 1e-3f;
      const int kq = rule.quota[kLevels - 1];
      if (rule.quantile ? kq <= kCand : target <= 0.99f) {
        auto mass_above = [&](float t, int* cnt) {
          float m = 0.f;
          int c = 0;
#pragma unroll
          for (int r = 0; r < K; ++r) {
            const bool in = lane * K + r < nvis && pj[r] >= t;
            m += in ? pj[r] : 0.f;
            c += in;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            m += __shfl_xor_sync(0xffffffffu, m, o);
            c += __shfl_xor_sync(0xffffffffu, c, o);
          }
          *cnt = c;
          return m;
        };
        float pmax = 0.f;
#pragma unroll
        for (int r = 0; r < K; ++r) pmax = fmaxf(pmax, pj[r]);
        pmax = warp_max(pmax);
        // do the blocks with P >= t reach past every kept rank?
        auto enough = [&](float t, int* cnt) {
          const float mass = mass_above(t, cnt);
          return rule.quantile ? *cnt >= kq : mass >= target;
        };
        int m_hi;
        float lo = 0.f, hi = pmax, t;
        int m;
        if (enough(hi, &m_hi)) {
          t = hi;
          m = m_hi;
        } else {
          int m_lo = nvis;                 // the whole row: mass 1 >= target, nvis >= K_3
          // stop as soon as the candidates fit (sorting them costs the same
          // for any count up to kCand)
          for (int it = 0; it < 40; ++it) {
            if (m_lo <= kCand) break;
            const float mid = 0.5f * (lo + hi);
            if (!(mid > lo && mid < hi)) break;
            int c;
            if (enough(mid, &c)) {
              lo = mid;
              m_lo = c;
            } else {
              hi = mid;
            }
          }
          t = lo;
          m = m_lo;
        }
        if (m <= kCand) {
          int mine = 0;
#pragma unroll
          for (int r = 0; r < K; ++r) mine += lane * K + r < nvis && pj[r] >= t;
          int tot;
          int pos = warp_excl_scan(mine, &tot);
#pragma unroll
          for (int r = 0; r < K; ++r) {
            const int i = lane * K + r;
            if (i < nvis && pj[r] >= t)
              key[pos++] = ((unsigned long long)__float_as_uint(pj[r]) << 32) | (0xffffffffu - (unsigned)i);
          }
          __syncwarp();
          // the candidates are a prefix of the ranking: sort them (P, then
          // lower index, descending; zero keys pad to a power of two) and give
          // each its level from its rank and the exclusive running mass
          unsigned long long v[kCandPerLane];
#pragma unroll
          for (int r = 0; r < kCandPerLane; ++r) {
            const int i = lane * kCandPerLane + r;
            v[r] = i < m ? key[i] : 0ull;
          }
          warp_bitonic_desc<kCandPerLane>(v);
          levels_from_sorted<kCandPerLane>(v, m, rule, lev);
          done = true;
        }
      }
    }
    if (!done) {
      // the whole row sorted in registers: lane L holds ranks L*K .. L*K + K - 1
      unsigned long long v[K];
#pragma unroll
      for (int r = 0; r < K; ++r) {
        const int i = lane * K + r;
        v[r] = i < nvis ? ((unsigned long long)__float_as_uint(pj[r]) << 32) | (0xffffffffu - (unsigned)i)
                        : 0ull;
      }
      warp_bitonic_desc<K>(v);
      levels_from_sorted<K>(v, nvis, rule, lev);
    }
  } else if constexpr (K < 0) {
    // Compact path of long rows: P of the visible blocks as floats.  The
    // candidate cut as below; a row whose cut does not fit ranks every block
    // against every other (exact; the launch takes this path only when the
    // cut is expected to fit).
    float* pv = reinterpret_cast<float*>(key);
    unsigned long long* cand = key + (((a.Nk + 31) & ~31) >> 1);
    for (int i = lane; i < nvis; i += 32) pv[i] = expf(z[i] - mx) * inv;
    __syncwarp();
    bool done = false;
    const float target = a.tau[kLevels - 1] + 1e-3f;
    const int kq = rule.quota[kLevels - 1];
    if (rule.quantile ? kq <= kCandS : target <= 0.99f) {
      auto enough = [&](float t, int* cnt) {
        float m = 0.f;
        int c = 0;
        for (int i = lane; i < nvis; i += 32) {
          const float pi = pv[i];
          const bool in = pi >= t;
          m += in ? pi : 0.f;
          c += in;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          m += __shfl_xor_sync(0xffffffffu, m, o);
          c += __shfl_xor_sync(0xffffffffu, c, o);
        }
        *cnt = c;
        return rule.quantile ? c >= kq : m >= target;
      };
      float pmax = 0.f;
      for (int i = lane; i < nvis; i += 32) pmax = fmaxf(pmax, pv[i]);
      pmax = warp_max(pmax);
      int m_hi, m;
      float lo = 0.f, hi = pmax, t;
      if (enough(hi, &m_hi)) {
        t = hi;
        m = m_hi;
      } else {
        int m_lo = nvis;
        for (int it = 0; it < 40; ++it) {
          if (m_lo <= kCandS) break;
          const float mid = 0.5f * (lo + hi);
          if (!(mid > lo && mid < hi)) break;
          int c;
          if (enough(mid, &c)) {
            lo = mid;
            m_lo = c;
          } else {
            hi = mid;
          }
        }
        t = lo;
        m = m_lo;
      }
      if (m <= kCandS) {
        int base = 0;
        for (int i0 = 0; i0 < nvis; i0 += 32) {
          const int i = i0 + lane;
          const float pi = i < nvis ? pv[i] : 0.f;
          const bool in = i < nvis && pi >= t;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (in)
            cand[base + __popc(bal & ((1u << lane) - 1))] =
                ((unsigned long long)__float_as_uint(pi) << 32) | (0xffffffffu - (unsigned)i);
          base += __popc(bal);
        }
        __syncwarp();
        unsigned long long v[kCandPerLaneS];
#pragma unroll
        for (int r = 0; r < kCandPerLaneS; ++r) {
          const int i = lane * kCandPerLaneS + r;
          v[r] = i < m ? cand[i] : 0ull;
        }
        warp_bitonic_desc<kCandPerLaneS>(v);
        levels_from_sorted<kCandPerLaneS>(v, m, rule, lev);
        done = true;
      }
    }
    if (!done) {
      // every block's rank (P descending, ties to the lower index) and the
      // mass ranked before it, by comparison with every other block
      for (int j = lane; j < nvis; j += 32) {
        const float pj = pv[j];
        float c = 0.f;
        int rank = 0;
        for (int i = 0; i < nvis; ++i) {
          const float pi = pv[i];
          const bool before = pi > pj || (pi == pj && i < j);
          c += before ? pi : 0.f;
          rank += before;
        }
        lev[j] = rule.level(c, rank);
      }
    }
  } else {
    for (int i = lane; i < n2; i += 32) key[i] = make_key(i);
    __syncwarp();
    // Candidate cut, as in the register path, over the keys in shared memory
    // (lane L reads keys L, L + 32, ...): blocks with P >= t are a prefix of
    // the ranking; t is bisected until they reach past every kept rank and
    // number at most kCandS, and only they are ranked.
    bool done = false;
    unsigned long long* cand = key + n2;
    const float target = a.tau[kLevels - 1] + 1e-3f;
    const int kq = rule.quota[kLevels - 1];
    if (rule.quantile ? kq <= kCandS : target <= 0.99f) {
      auto pk = [](unsigned long long k) { return __uint_as_float((unsigned)(k >> 32)); };
      auto enough = [&](float t, int* cnt) {
        float m = 0.f;
        int c = 0;
        for (int i = lane; i < nvis; i += 32) {
          const float pi = pk(key[i]);
          const bool in = pi >= t;
          m += in ? pi : 0.f;
          c += in;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          m += __shfl_xor_sync(0xffffffffu, m, o);
          c += __shfl_xor_sync(0xffffffffu, c, o);
        }
        *cnt = c;
        return rule.quantile ? c >= kq : m >= target;
      };
      float pmax = 0.f;
      for (int i = lane; i < nvis; i += 32) pmax = fmaxf(pmax, pk(key[i]));
      pmax = warp_max(pmax);
      int m_hi, m;
      float lo = 0.f, hi = pmax, t;
      if (enough(hi, &m_hi)) {
        t = hi;
        m = m_hi;
      } else {
        int m_lo = nvis;
        for (int it = 0; it < 40; ++it) {
          if (m_lo <= kCandS) break;
          const float mid = 0.5f * (lo + hi);
          if (!(mid > lo && mid < hi)) break;
          int c;
          if (enough(mid, &c)) {
            lo = mid;
            m_lo = c;
          } else {
            hi = mid;
          }
        }
        t = lo;
        m = m_lo;
      }
      if (m <= kCandS) {
        // compact the candidates (in index order; the ranking below needs no order)
        int base = 0;
        for (int i0 = 0; i0 < nvis; i0 += 32) {
          const int i = i0 + lane;
          const unsigned long long ki = i < nvis ? key[i] : 0ull;
          const bool in = i < nvis && pk(ki) >= t;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (in) cand[base + __popc(bal & ((1u << lane) - 1))] = ki;
          base += __popc(bal);
        }
        __syncwarp();
        // sort the candidates in registers and scan, as in the register path
        unsigned long long v[kCandPerLaneS];
#pragma unroll
        for (int r = 0; r < kCandPerLaneS; ++r) {
          const int i = lane * kCandPerLaneS + r;
          v[r] = i < m ? cand[i] : 0ull;
        }
        warp_bitonic_desc<kCandPerLaneS>(v);
        levels_from_sorted<kCandPerLaneS>(v, m, rule, lev);
        done = true;
      }
    }
    if (!done) {
    // bitonic sort in shared memory, descending: P high, then lower index first
    for (int k = 2; k <= n2; k <<= 1) {
      for (int sd = k >> 1; sd > 0; sd >>= 1) {
        for (int i = lane; i < n2; i += 32) {
          const int ixj = i ^ sd;
          if (ixj > i) {
            const unsigned long long u = key[i], w = key[ixj];
            const bool desc = (i & k) == 0;
            if (desc ? (u < w) : (u > w)) { key[i] = w; key[ixj] = u; }
          }
        }
        __syncwarp();
      }
    }
    const int per = (nvis + 31) / 32;       // lanes take contiguous rank ranges
    const int r0 = lane * per, r1 = min(nvis, r0 + per);
    float mine = 0.f;
    for (int r = r0; r < r1; ++r) mine += __uint_as_float((unsigned)(key[r] >> 32));
    float total;
    float c = warp_excl_scan(mine, &total);
    for (int r = r0; r < r1; ++r) {
      const float pr = __uint_as_float((unsigned)(key[r] >> 32));
      const int j = (int)(0xffffffffu - (unsigned)(key[r] & 0xffffffffu));
      lev[j] = rule.level(c, r);
      c += pr;
    }
    }
  }
  __syncwarp();
  // overrides: causal diagonal -> 0, forced prefix -> 0 (visible blocks only)
  for (int j = lane; j < nvis; j += 32) {
    const bool strad = a.causal && (min((j + 1) * a.kv_blk, a.N) - 1 >= q_lo);
    const bool forced = j * a.kv_blk < a.forced_prefix_tokens;
    if (strad || forced) lev[j] = 0;
  }
  __syncwarp();
  if (a.sim_threshold > -1.f) {
    // cosine-similarity constraint: a kept block's level is lowered to the
    // largest its KV head's merges allow (pruned blocks stay pruned)
    const int bhq = row / a.Nq;
    const int bhk = (bhq / a.Hq) * a.Hkv + (bhq % a.Hq) / (a.Hq / a.Hkv);
    const int8_t* ml = maxlev + (long long)bhk * a.Nk;
    for (int j = lane; j < a.Nk; j += 32)
      if (lev[j] > ml[j]) lev[j] = ml[j];
    __syncwarp();
  }
  int8_t* mrow = map_ws + (long long)row * a.Nk;
  for (int j = lane; j < a.Nk; j += 32) {
    mrow[j] = lev[j];
    if (map_user) map_user[(long long)row * a.Nk + j] = lev[j];
    if (mass_user) mass_user[(long long)row * a.Nk + j] = j < nvis ? expf(z[j] - mx) * inv : 0.f;
  }
  emit_list_warp(lev, a.Nk, list + (long long)row * a.Nk, counts + row);
}

// A caller's level map -> the work list.  The map is held to the method's
// contract first: a value outside -1..3 counts as pruned; causally, a block
// after the query block's last row is pruned and a kept block straddling its
// diagonal is attended at level 0 (with the token mask), since a pooled key
// there would average future tokens.  Every changed entry sets kErrLevelMap in
// the workspace error word (psa_check_device reports it).
__global__ void map_to_list_kernel(MaskArgs a, int rows_per_cta, int nrows,
                                   const int8_t* __restrict__ map, int* __restrict__ list,
                                   int4* __restrict__ counts, int* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * rows_per_cta + warp;
  if (row >= nrows) return;
  const int lev_stride = (a.Nk + 15) & ~15;
  int8_t* lev = reinterpret_cast<int8_t*>(smem) + (size_t)warp * lev_stride;
  const int q_lo = (row % a.Nq) * a.q_blk;
  const int q_hi = min(a.N, q_lo + a.q_blk) - 1;
  bool changed = false;
  for (int j = lane; j < lev_stride; j += 32) {
    const int8_t v = j < a.Nk ? map[(long long)row * a.Nk + j] : (int8_t)-1;
    int8_t u = (v >= -1 && v < kLevels) ? v : (int8_t)-1;
    if (a.causal && j < a.Nk) {
      if (j * a.kv_blk > q_hi) u = -1;                                        // future block
      else if (u > 0 && min((j + 1) * a.kv_blk, a.N) - 1 >= q_lo) u = 0;   // straddles
    }
    changed |= j < a.Nk && u != v;
    lev[j] = u;
  }
  if (__any_sync(0xffffffffu, changed) && lane == 0) atomicOr(err, kErrLevelMap);
  __syncwarp();
  emit_list_warp(lev, a.Nk, list + (long long)row * a.Nk, counts + row);
}

#ifdef PSA_DEBUG
// Debug builds only: every consumer of a work list reads entries by index and
// turns them into addresses, so a list that no kernel of this library wrote
// (a corrupted workspace) is checked first.  A row whose counts are negative
// or add up to more than Nk, or whose entries leave [0, Nk) or are not
// increasing inside a level, is reported in the error word (kErrListBounds)
// and emptied (its counts set to 0), so that no kernel reads through it.
__global__ void list_check_kernel(MaskArgs a, int nrows, const int* __restrict__ list,
                                  int4* __restrict__ counts, int* __restrict__ err) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= nrows) return;
  const int4 c = counts[row];
  const long long tot = (long long)c.x + c.y + c.z + c.w;
  bool bad = c.x < 0 || c.y < 0 || c.z < 0 || c.w < 0 || tot > a.Nk;
  if (!bad) {
    const int* lrow = list + (long long)row * a.Nk;
    const int f1 = c.x, f2 = f1 + c.y, f3 = f2 + c.z;
    for (int e = lane; e < (int)tot; e += 32) {
      const int j = lrow[e];
      const bool first = e == 0 || e == f1 || e == f2 || e == f3;
      bad |= j < 0 || j >= a.Nk || (!first && j <= lrow[e - 1]);
    }
    bad = __any_sync(0xffffffffu, bad);
  }
  if (bad && lane == 0) {
    counts[row] = make_int4(0, 0, 0, 0);
    atomicOr(err, kErrListBounds);
  }
}
#endif

int next_pow2(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

}  // namespace

cudaError_t launch_qmean(const psa_params_t& p, const Layout& L, const void* Q, char* ws,
                         cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, 0.f);
  const int grid = p.B * p.Hq * L.Nq;
  const int threads = p.q_blk * p.d / 64;  // 8 rows per thread: 64 to 256 threads
  float* qh = (float*)(ws + L.qmh);
  float* ql = (float*)(ws + L.qml);
  if (p.dtype == PSA_BF16)
    return launch_dependent(qmean_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, st, a,
                            (const __nv_bfloat16*)Q, qh, ql);
  return launch_dependent(qmean_kernel<float>, dim3(grid), dim3(threads), 0, st, a,
                          (const float*)Q, qh, ql);
}

cudaError_t launch_assign(const psa_params_t& p, const Layout& L, float scale, char* ws,
                          int8_t* user_map, float* block_mass, cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, scale);
  const int n2 = next_pow2(L.Nk < 32 ? 32 : L.Nk);
  const bool in_regs = n2 <= 1024;          // register sort; larger rows sort in shared memory
  // Long rows: the compact path (P as floats, a candidate set), unless the
  // candidate cut cannot apply (a last threshold within 1% of the whole mass,
  // or a quantile quota past the candidate set), where every row sorts all
  // its keys.
  const int quota3 = (int)ceil((double)p.tau[kLevels - 1] * (double)L.Nk);
  const bool cut = p.assign == PSA_ASSIGN_QUANTILE ? quota3 <= kCandS
                                                    : p.tau[kLevels - 1] + 1e-3f <= 0.99f;
  const int K = in_regs ? n2 / 32 : (cut ? -1 : 0);
  const size_t per_row = assign_key_bytes(K, n2, L.Nk) + ((L.Nk + 15) & ~15);
  int rows_per_cta = (int)((96 * 1024) / per_row);
  rows_per_cta = rows_per_cta < 1 ? 1 : (rows_per_cta > 2 ? 2 : rows_per_cta);
  const size_t smem = per_row * rows_per_cta;
  const int nrows = p.B * p.Hq * L.Nq;
  const int grid = (nrows + rows_per_cta - 1) / rows_per_cta;
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3(grid), dim3(32 * rows_per_cta), smem, st, a, n2,
                            rows_per_cta, nrows, (const float*)(ws + L.zlog),
                            (const int8_t*)(ws + L.maxlev), (int8_t*)(ws + L.map), user_map,
                            block_mass, (int*)(ws + L.list), (int4*)(ws + L.counts));
  };
  switch (n2) {   // keys per lane for the register sort; larger rows sort in shared memory
    case 32: return go(assign_kernel<1>);
    case 64: return go(assign_kernel<2>);
    case 128: return go(assign_kernel<4>);
    case 256: return go(assign_kernel<8>);
    case 512: return go(assign_kernel<16>);
    case 1024: return go(assign_kernel<32>);
    default: return K < 0 ? go(assign_kernel<-1>) : go(assign_kernel<0>);
  }
}

cudaError_t launch_list_check(const psa_params_t& p, const Layout& L, char* ws, cudaStream_t st) {
#ifdef PSA_DEBUG
  const MaskArgs a = make_mask_args(p, L, 0.f);
  const int nrows = p.B * p.Hq * L.Nq;
  return launch_dependent(list_check_kernel, dim3((nrows + 7) / 8), dim3(256), 0, st, a, nrows,
                          (const int*)(ws + L.list), (int4*)(ws + L.counts), (int*)(ws + L.err));
#else
  (void)p; (void)L; (void)ws; (void)st;
  return cudaSuccess;
#endif
}

cudaError_t launch_map_to_list(const psa_params_t& p, const Layout& L, const int8_t* map,
                               char* ws, cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, 0.f);
  const int rows_per_cta = 8;
  const size_t smem = (size_t)((L.Nk + 15) & ~15) * rows_per_cta;
  cudaError_t e = cudaFuncSetAttribute(map_to_list_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nrows = p.B * p.Hq * L.Nq;
  return launch_dependent(map_to_list_kernel, dim3((nrows + rows_per_cta - 1) / rows_per_cta),
                          dim3(32 * rows_per_cta), smem, st, a, rows_per_cta, nrows, map,
                          (int*)(ws + L.list), (int4*)(ws + L.counts), (int*)(ws + L.err));
}

}  // namespace psa
