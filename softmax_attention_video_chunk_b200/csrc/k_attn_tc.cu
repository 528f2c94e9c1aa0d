// Window + anchor Softmax attention on the sm_100a tensor cores.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method, the paragraph on the local window: exact Softmax over the
// chunk-aligned window plus the two boundary anchors (four-way
// connectivity), each key once.  The pages run this through a varlen
// FlashAttention call with queries packed by visible-key pattern; here one
// CTA owns two 128-row query tiles of one visible-key group (Geo::group) and
// walks that group's key ranges directly.
//
// Per CTA (320 threads, one CTA per SM):
//   warp 8      TMA producer: Q tiles once, then K (bf16) and V^T (fp16) tiles
//               of 128 keys into a 2-stage ring;
//   warp 9      MMA issuer (one thread): S_j = Q_j K^T (bf16, FP32 in TMEM),
//               O_j += P_j V (P fp16 read from TMEM, V^T from smem);
//   warps 0-3   softmax of query tile 0, warps 4-7 of tile 1: one thread per
//               row reads its S row from TMEM, applies the key-range mask,
//               keeps a running max (rescaling O in TMEM only when the max grows
//               by more than 2^8) and row sum, writes P = 2^(s - m) as fp16
//               over its S columns, and finally normalises O and writes
//               g_s * o_s (fp16, the projection operand) or o_s (fp32).
// Text queries (n_qtext > 0): the same kernel runs the text tokens' rows as
// one dense group over every video key plus the text keys (o_s output only).
// TMEM (512 columns): S0 | S1 | O0 | O1.  Every mbarrier wait is bounded in
// time; on expiry the CTA records VDN_ERR_TIMEOUT in the status word, drains
// its MMAs and copies, frees TMEM and exits.
#include <math.h>

#include "mx_encode.cuh"
#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_tc.h"

namespace vdn {

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

struct Abort {
  volatile int* flag;
  int* status;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Abort& ab) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*ab.flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *ab.flag = 1;
      atomicOr(ab.status, kDevTimeout);
      return false;
    }
  }
}

constexpr int kBK = 128;  // keys per tile
// Of every 8 (key-pair) exponentials of a full tile, this many are evaluated
// on the FMA pipe (polynomial) and the rest on the MUFU pipe, so that neither
// pipe limits the softmax warps.
#ifndef VDN_KEMU
#define VDN_KEMU 2
#endif
constexpr int kEmu = VDN_KEMU;

// Key tile i of a group: tiles of each key range start at the range start
// rounded down to 8 tokens (16-byte TMA coordinate of V^T); columns outside
// [lo, hi) belong to no range of this group and are masked.
__device__ __forceinline__ void kv_tile(const QGroup& g, int i, int& k0, int& lo, int& hi) {
  k0 = 0; lo = 0; hi = 0;
  bool found = false;
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    if (s < g.nseg && !found) {
      const int a = g.seg0[s] & ~7;
      const int nt = (g.seg1[s] - a + kBK - 1) / kBK;
      if (i < nt) {
        k0 = a + i * kBK;
        lo = max(g.seg0[s], k0) - k0;
        hi = min(g.seg1[s], k0 + kBK) - k0;
        found = true;
      } else {
        i -= nt;
      }
    }
  }
}

__device__ __forceinline__ int kv_count(const QGroup& g) {
  int n = 0;
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    if (s < g.nseg) {
      const int a = g.seg0[s] & ~7;
      n += (g.seg1[s] - a + kBK - 1) / kBK;
    }
  }
  return n;
}

// Tile i of a query group's key sequence: the group's video key tiles, then
// (when text keys join the Softmax) ceil(n_text / kBK) tiles of text tokens.
__device__ __forceinline__ void kv_tile_all(const QGroup& g, int n_video, int n_text, int i,
                                            int& k0, int& lo, int& hi, bool& text) {
  text = i >= n_video;
  if (!text) {
    kv_tile(g, i, k0, lo, hi);
  } else {
    k0 = (i - n_video) * kBK;
    lo = 0;
    hi = min(kBK, n_text - k0);
  }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace

template <int D, bool FUSED>
__global__ void __launch_bounds__(320, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_vt,
               const __grid_constant__ CUtensorMap map_tk,
               const __grid_constant__ CUtensorMap map_tvt, int n_text, Geo geo, int B, int H,
               float scale_log2, const __nv_bfloat16* __restrict__ gates,
               __half* __restrict__ x, uint8_t* __restrict__ xq, uint8_t* __restrict__ sfa,
               float* __restrict__ o_s, int* __restrict__ status,
               int n_qtext, int kv_split, float* __restrict__ ml) {
  constexpr int BM = 128, NS = 2;
  constexpr int QT = BM * D * 2;   // bytes of a Q tile
  constexpr int KT = kBK * D * 2;  // bytes of a K tile
  constexpr int VT = kBK * D * 2;  // bytes of a V^T tile
  constexpr int NSUB = D / 64;     // 128-byte column panels of a Q / K row

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 2 * QT;
  uint8_t* sV = sK + NS * KT;
  uint64_t* bars = (uint64_t*)(sV + NS * VT);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint64_t* p_half = drain + 1;  // first 64 keys of P_j stored
  uint32_t* tmem_slot = (uint32_t*)(p_half + 2);
  int* abort_flag = (int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * H;
  // kv_split > 1 (text rows only): CTA `split` of a row pair walks its share
  // of the key tiles and writes a partial result (o normalised by its own sum,
  // plus the running max and sum) for a combine pass
  const int pq = blockIdx.x / BH, bh = blockIdx.x % BH;
  const int pair = pq / kv_split, split = pq % kv_split;
  const int b = bh / H, h = bh % H;
  QGroup g;
  int row0;
  if (n_qtext > 0) {  // text queries: one dense group over every video key
    g.row0 = 0; g.nrows = n_qtext; g.nseg = 1;
    g.seg0[0] = 0; g.seg1[0] = geo.T * geo.N;
    g.seg0[1] = g.seg1[1] = g.seg0[2] = g.seg1[2] = 0;
    row0 = pair * 2 * BM;
    if (row0 >= n_qtext) return;  // uniform over the CTA
  } else if (!find_tile(geo, 2 * BM, pair, &g, &row0)) {
    return;  // uniform over the CTA
  }
  const int row_end = g.row0 + g.nrows;
  const bool has1 = row0 + BM < row_end;
  const int n_video = kv_count(g);
  const int n_all = n_video + (n_text + kBK - 1) / kBK;
  const int kv0 = (int)((long long)n_all * split / kv_split);  // this CTA: tiles kv0 ..
  const int n_kv = (int)((long long)n_all * (split + 1) / kv_split) - kv0;
  const int L = geo.T * geo.N;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(k_full + i, 1);
      ptx::mbar_init(v_full + i, 1);
      ptx::mbar_init(kv_empty + i, 1);
    }
    for (int j = 0; j < 2; ++j) {
      ptx::mbar_init(s_full + j, 1);
      ptx::mbar_init(p_full + j, 128);
      ptx::mbar_init(p_half + j, 128);
      ptx::mbar_init(o_done + j, 1);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, status};

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&map_q);
      ptx::prefetch_tmap(&map_k);
      ptx::prefetch_tmap(&map_vt);
      if (n_text > 0) {
        ptx::prefetch_tmap(&map_tk);
        ptx::prefetch_tmap(&map_tvt);
      }
      ptx::mbar_arrive_expect_tx(q_full, (has1 ? 2 : 1) * QT);
      for (int j = 0; j < (has1 ? 2 : 1); ++j)
        for (int sub = 0; sub < NSUB; ++sub)
          ptx::tma_load_4d(sQ + j * QT + sub * BM * 128, &map_q, q_full, sub * 64, h,
                           row0 + j * BM, b);
      int issued = 0;
      for (int i = 0; i < n_kv; ++i) {
        const int st = i % NS, use = i / NS;
        if (use > 0 && !wait_bar(kv_empty + st, (use - 1) & 1, ab)) break;
        int k0, lo, hi;
        bool text;
        kv_tile_all(g, n_video, n_text, kv0 + i, k0, lo, hi, text);
        const CUtensorMap* mk = text ? &map_tk : &map_k;
        const CUtensorMap* mv = text ? &map_tvt : &map_vt;
        ptx::mbar_arrive_expect_tx(k_full + st, KT);
        for (int sub = 0; sub < NSUB; ++sub)
          ptx::tma_load_4d(sK + st * KT + sub * kBK * 128, mk, k_full + st, sub * 64, h, k0, b);
        ptx::mbar_arrive_expect_tx(v_full + st, VT);
        for (int vs = 0; vs < 2; ++vs)
          ptx::tma_load_3d(sV + st * VT + vs * D * 128, mv, v_full + st, k0 + vs * 64, 0, bh);
        issued = i + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA releases its smem
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int i = max(0, issued - NS); i < issued; ++i) {
          const int st = i % NS, ph = (i / NS) & 1;
          while (!ptx::mbar_try_wait(k_full + st, ph) && ptx::globaltimer_ns() - t0 < kWaitLimitNs) {}
          while (!ptx::mbar_try_wait(v_full + st, ph) && ptx::globaltimer_ns() - t0 < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = ptx::idesc_f16(128, kBK, 1);
      constexpr uint32_t idO = ptx::idesc_f16(128, D, 0);
      const uint32_t sQa = ptx::smem_u32(sQ), sKa = ptx::smem_u32(sK), sVa = ptx::smem_u32(sV);
      auto issue_S = [&](int j, int st) {
        const uint32_t d = tmem + j * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint64_t a = ptx::sdesc_k_sw128(sQa + j * QT + off);
          const uint64_t bd = ptx::sdesc_k_sw128(sKa + st * KT + (kk >> 2) * (kBK * 128) + (kk & 3) * 32);
          ptx::mma_ss(d, a, bd, idS, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(s_full + j);
      };
      // O_j += P_j V over key slices kk0 .. kk1-1 (16 keys each); the first
      // half runs as soon as the softmax warps have stored P's first 64 keys
      auto issue_PV = [&](int j, int st, bool first, int kk0, int kk1) {
        const uint32_t d = tmem + 256 + j * D;
        const uint32_t pa = tmem + j * 128;
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk) {
          const uint64_t bd = ptx::sdesc_k_sw128(sVa + st * VT + (kk >> 2) * (D * 128) + (kk & 3) * 32);
          ptx::mma_ts(d, pa + kk * 8, bd, idO, (!first || kk > 0) ? 1u : 0u);
        }
      };
      auto issue_PV_tile = [&](int j, int st, bool first, uint32_t ph) -> bool {
        if (!wait_bar(p_half + j, ph, ab)) return false;
        ptx::tc_fence_after();
        issue_PV(j, st, first, 0, kBK / 32);
        if (!wait_bar(p_full + j, ph, ab)) return false;
        ptx::tc_fence_after();
        issue_PV(j, st, first, kBK / 32, kBK / 16);
        ptx::mma_commit(o_done + j);
        return true;
      };
      bool ok = wait_bar(q_full, 0, ab) && wait_bar(k_full, 0, ab);
      if (ok) {
        ptx::tc_fence_after();
        issue_S(0, 0);
        if (has1) issue_S(1, 0);
      }
      for (int i = 0; ok && i < n_kv; ++i) {
        const int st = i % NS, ph = (i / NS) & 1;
        const int st2 = (i + 1) % NS, ph2 = ((i + 1) / NS) & 1;
        if (!(ok = wait_bar(v_full + st, ph, ab))) break;
        if (!(ok = issue_PV_tile(0, st, i == 0, i & 1))) break;
        if (i + 1 < n_kv) {
          if (!(ok = wait_bar(k_full + st2, ph2, ab))) break;
          ptx::tc_fence_after();
          issue_S(0, st2);
        }
        if (has1 && !(ok = issue_PV_tile(1, st, i == 0, i & 1))) break;
        ptx::mma_commit(kv_empty + st);
        if (has1 && i + 1 < n_kv) issue_S(1, st2);
      }
      // every MMA of this CTA completes before TMEM is released
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < kWaitLimitNs) {}
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int j = warp >> 2, wq = warp & 3;
    if (j == 0 || has1) {
      const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
      const uint32_t tS = tmem + lane_off + j * 128;
      const uint32_t tO = tmem + lane_off + 256 + j * D;
      float m_used = -INFINITY, l_sum = 0.f;
      bool ok = true;
      for (int i = 0; i < n_kv; ++i) {
        int k0, lo, hi;
        bool text;
        kv_tile_all(g, n_video, n_text, kv0 + i, k0, lo, hi, text);
        if (!(ok = wait_bar(s_full + j, i & 1, ab))) break;
        ptx::tc_fence_after();
        // pass 1: row maximum (all four 32-column loads in flight at once)
        const bool full = (lo == 0 && hi == kBK);  // tile wholly inside one key range
        float mx;
        {
          uint32_t s[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]);
            ptx::tmem_ld32(tS + 32 * c, chunk);
          }
          ptx::tmem_wait_ld();
          if (full) {
            // eight independent max chains, then a short tree
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = fmaxf(__uint_as_float(s[u]), __uint_as_float(s[8 + u]));
#pragma unroll
            for (int e = 16; e < 128; e += 16)
#pragma unroll
              for (int u = 0; u < 8; ++u)
                m8[u] = ptx::max3(m8[u], __uint_as_float(s[e + u]), __uint_as_float(s[e + 8 + u]));
            const float mr = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mx = mr * scale_log2;  // scale_log2 > 0
          } else {
            float mr = -INFINITY;
#pragma unroll
            for (int e = 0; e < 128; ++e)
              if (e >= lo && e < hi) mr = fmaxf(mr, __uint_as_float(s[e]));
            mx = mr * scale_log2;
          }
        }
        if (i == 0) {
          m_used = mx;
        } else {
          const bool need = mx > m_used + 8.f;
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = fmaxf(m_used, mx);
            const float f = ptx::ex2(m_used - m_new);
            l_sum *= f;
            m_used = m_new;
            if (!(ok = wait_bar(o_done + j, (i - 1) & 1, ab))) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              ptx::tmem_ld32(tO + 32 * c, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              ptx::tmem_st32(tO + 32 * c, o);
            }
            ptx::tmem_wait_st();
          }
        }
        // pass 2: P = 2^(s*scale - m) as fp16 pairs over the first 64 columns of S
        const float neg_m = -m_used;
        const uint64_t c2 = ptx::f2_pack(scale_log2, scale_log2);
        const uint64_t nm2 = ptx::f2_pack(neg_m, neg_m);
        uint64_t acc4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) acc4[u] = ptx::f2_pack(0.f, 0.f);
        if (full) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[64], pk[32];
            uint32_t (&ra)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
            uint32_t (&rb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
            ptx::tmem_ld32(tS + 64 * half, ra);
            ptx::tmem_ld32(tS + 64 * half + 32, rb);
            if (half == 1) {  // P's first 64 keys are stored: PV may start on them
              ptx::tmem_wait_st();
              ptx::tc_fence_before();
              ptx::mbar_arrive(p_half + j);
            }
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint64_t x2 = ptx::f2_fma(
                  ptx::f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), c2, nm2);
              uint64_t p2;
              if ((e & 7) < kEmu) {  // FMA-pipe exponentials
                p2 = ptx::exp2_poly2(x2);
              } else {               // MUFU exponentials
                float x0, x1;
                ptx::f2_unpack(x2, x0, x1);
                p2 = ptx::f2_pack(ptx::ex2(x0), ptx::ex2(x1));
              }
              acc4[e & 3] = ptx::f2_add(acc4[e & 3], p2);
              float p0, p1;
              ptx::f2_unpack(p2, p0, p1);
              pk[e] = pack_half2(p0, p1);
            }
            ptx::tmem_st32(tS + 32 * half, pk);
          }
        } else {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[64], pk[32];
            uint32_t (&ra)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
            uint32_t (&rb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
            ptx::tmem_ld32(tS + 64 * half, ra);
            ptx::tmem_ld32(tS + 64 * half + 32, rb);
            if (half == 1) {  // P's first 64 keys are stored: PV may start on them
              ptx::tmem_wait_st();
              ptx::tc_fence_before();
              ptx::mbar_arrive(p_half + j);
            }
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = 64 * half + 2 * e;
              float x0, x1;
              ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(r[2 * e]),
                                                      __uint_as_float(r[2 * e + 1])), c2, nm2),
                             x0, x1);
              const float p0 = (col >= lo && col < hi) ? ptx::ex2(x0) : 0.f;
              const float p1 = (col + 1 >= lo && col + 1 < hi) ? ptx::ex2(x1) : 0.f;
              acc4[e & 3] = ptx::f2_add(acc4[e & 3], ptx::f2_pack(p0, p1));
              pk[e] = pack_half2(p0, p1);
            }
            ptx::tmem_st32(tS + 32 * half, pk);
          }
        }
        float sum;
        {
          float s0, s1;
          ptx::f2_unpack(ptx::f2_add(ptx::f2_add(acc4[0], acc4[1]), ptx::f2_add(acc4[2], acc4[3])),
                         s0, s1);
          sum = s0 + s1;
        }
        ptx::tmem_wait_st();
        l_sum += sum;
        ptx::tc_fence_before();
        ptx::mbar_arrive(p_full + j);
      }
      if (ok && n_kv > 0 && wait_bar(o_done + j, (n_kv - 1) & 1, ab)) {
        ptx::tc_fence_after();
        const int row = row0 + j * BM + wq * 32 + lane;
        const bool valid = row < row_end;
        const float inv = 1.f / l_sum;
        const size_t tok = (size_t)b * (n_qtext > 0 ? n_qtext : L) + row;
        bool bad = false;
        float* o_out = o_s;
        if (kv_split > 1) {  // partial result of this key share
          const size_t rows_all = (size_t)B * n_qtext * H;
          o_out = o_s + (size_t)split * rows_all * D;
          if (valid) {
            float* mlp = ml + ((size_t)split * rows_all + tok * H + h) * 2;
            mlp[0] = m_used;
            mlp[1] = l_sum;
          }
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + 32 * c, o);
          ptx::tmem_wait_ld();
          if (!valid) continue;
          if constexpr (FUSED) {
            const uint4* gp = reinterpret_cast<const uint4*>(gates + (tok * H + h) * D + 32 * c);
            uint32_t hw[16];  // g_s * o_s of this 32-column block, fp16
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const uint4 gg = gp[v4];
              const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gg);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 gf = __bfloat1622float2(g2[e]);
                const float a0 = gf.x * __uint_as_float(o[8 * v4 + 2 * e]) * inv;
                const float a1 = gf.y * __uint_as_float(o[8 * v4 + 2 * e + 1]) * inv;
                bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
                hw[4 * v4 + e] = pack_half2(a0, a1);
              }
            }
            const size_t K = (size_t)(2 * H * D);
            if (xq == nullptr) {
              uint4* xp = reinterpret_cast<uint4*>(x + tok * K + (size_t)h * D + 32 * c);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                xp[v4] = make_uint4(hw[4 * v4], hw[4 * v4 + 1], hw[4 * v4 + 2], hw[4 * v4 + 3]);
            } else {  // the same fp16 values, quantised to MXFP8 (one 32-element block)
              uint32_t cw[8];
              const uint32_t eb = mx::encode32(hw, cw);
              uint4* qp = reinterpret_cast<uint4*>(xq + tok * K + (size_t)h * D + 32 * c);
              qp[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
              qp[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
              sfa[mx::sf_offset(tok, (h * D + 32 * c) / 32, (int)K)] = (uint8_t)eb;
            }
          } else {
            float4* op = reinterpret_cast<float4*>(o_out + (tok * H + h) * D + 32 * c);
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              op[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv, __uint_as_float(o[4 * v4 + 1]) * inv,
                                   __uint_as_float(o[4 * v4 + 2]) * inv, __uint_as_float(o[4 * v4 + 3]) * inv);
          }
        }
        if (bad) atomicOr(status, kDevRange);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 9) ptx::tmem_dealloc(tmem, 512);
}

// Text rows split over key shares: o = sum_s w_s o_s / sum_s w_s with
// w_s = l_s 2^(m_s - max_s m_s) (o_s normalised by its own sum l_s, m_s the
// running maximum in log2 units).  One warp per (token, head) row.
template <int D>
__global__ void __launch_bounds__(256)
combine_splits_kernel(const float* __restrict__ part, const float* __restrict__ ml,
                      float* __restrict__ out, size_t rows, int S) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, ml[((size_t)s * rows + r) * 2]);
  float W = 0.f, acc[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
  for (int s = 0; s < S; ++s) {
    const float* m2 = ml + ((size_t)s * rows + r) * 2;
    const float w = m2[1] * exp2f(m2[0] - M);
    W += w;
    const float* p = part + ((size_t)s * rows + r) * D + lane * CPL;
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = fmaf(w, p[i], acc[i]);
  }
  const float inv = 1.f / W;
#pragma unroll
  for (int i = 0; i < CPL; ++i) out[r * D + lane * CPL + i] = acc[i] * inv;
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

template <int D, bool FUSED>
static cudaError_t launch_attn_t(const TcAttnArgs& t, const TcFwdArgs* f, float* o_s,
                                 cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const uint64_t L = t.L, H = t.H, B = t.B;
  {
    const uint64_t dims[4] = {(uint64_t)D, H, L, B};
    const uint64_t str[3] = {(uint64_t)D * 2, H * D * 2, L * H * D * 2};
    const uint32_t box[4] = {64, 1, 128, 1};
    if (!make_tmap(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.k, dims, str, box))
      return cudaErrorInvalidValue;
    if (t.text_q == nullptr &&
        !make_tmap(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.q, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const int n_qtext = t.text_q != nullptr ? t.n_text_keys : 0;
  if (n_qtext > 0) {  // queries are the text tokens [B, n_text, H, D]
    const uint64_t nt = (uint64_t)n_qtext;
    const uint64_t dims[4] = {(uint64_t)D, H, nt, B};
    const uint64_t str[3] = {(uint64_t)D * 2, H * D * 2, nt * H * D * 2};
    const uint32_t box[4] = {64, 1, 128, 1};
    if (!make_tmap(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.text_q, dims, str, box))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)t.Lp, (uint64_t)D, B * H};
    const uint64_t str[2] = {(uint64_t)t.Lp * 2, (uint64_t)D * t.Lp * 2};
    const uint32_t box[3] = {64, (uint32_t)D, 1};
    if (!make_tmap(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, t.vt, dims, str, box))
      return cudaErrorInvalidValue;
  }
  CUtensorMap mtk = mk, mtv = mv;  // stand-ins when no text keys (never read)
  if (t.n_text_keys > 0) {
    const uint64_t nt = (uint64_t)t.n_text_keys;
    const uint64_t dims[4] = {(uint64_t)D, H, nt, B};
    const uint64_t str[3] = {(uint64_t)D * 2, H * D * 2, nt * H * D * 2};
    const uint32_t box[4] = {64, 1, 128, 1};
    if (!make_tmap(&mtk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.text_k, dims, str, box))
      return cudaErrorInvalidValue;
    const uint64_t dv[3] = {(uint64_t)t.ntp, (uint64_t)D, B * H};
    const uint64_t sv[2] = {(uint64_t)t.ntp * 2, (uint64_t)D * t.ntp * 2};
    const uint32_t bv[3] = {64, (uint32_t)D, 1};
    if (!make_tmap(&mtv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, t.vt_text, dv, sv, bv))
      return cudaErrorInvalidValue;
  }
  Geo geo{t.T, t.N, t.C, t.R};
  const int kv_split = (n_qtext > 0 && t.part != nullptr && t.kv_split > 1) ? t.kv_split : 1;
  const int pairs =
      (n_qtext > 0 ? (n_qtext + 255) / 256 : count_tiles(geo, 256)) * kv_split;
  const size_t sm = 1024 + 2 * (128 * D * 2) + 2 * 2 * (128 * D * 2) + 256;
  auto kern = attn_tc_kernel<D, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const float scale_log2 = t.scale * 1.4426950408889634f;
  const unsigned grid = (unsigned)pairs * (unsigned)(t.B * t.H);
  kern<<<grid, 320, sm, st>>>(mq, mk, mv, mtk, mtv, t.n_text_keys, geo, t.B, t.H, scale_log2,
                              FUSED ? (const __nv_bfloat16*)f->gates : nullptr,
                              FUSED ? f->x : nullptr, FUSED ? f->xq : nullptr,
                              FUSED ? f->sfa : nullptr, kv_split > 1 ? t.part : o_s, t.status,
                              n_qtext, kv_split, t.ml);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (kv_split > 1) {
    const size_t rows = (size_t)t.B * n_qtext * t.H;
    combine_splits_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(t.part, t.ml, o_s, rows,
                                                                           kv_split);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_attn_tc(const TcAttnArgs& t, const TcFwdArgs* f, float* o_s, cudaStream_t st) {
  if (f != nullptr && t.text_q != nullptr) return cudaErrorInvalidValue;  // text rows: o_s only
  if (f != nullptr) {
    if (t.D == 128) return launch_attn_t<128, true>(t, f, nullptr, st);
    if (t.D == 64) return launch_attn_t<64, true>(t, f, nullptr, st);
  } else {
    if (t.D == 128) return launch_attn_t<128, false>(t, nullptr, o_s, st);
    if (t.D == 64) return launch_attn_t<64, false>(t, nullptr, o_s, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
