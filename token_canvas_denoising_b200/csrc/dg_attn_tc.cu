// Bidirectional GQA canvas attention on the 5th-generation tensor cores.
//
// Method: every canvas position attends to every other canvas position (no
// triangular mask) and to the prompt's cached K/V ("DiffusionGemma解析：扩散模型如何
// 让LLM快5倍", 整片并行去噪, last paragraph; "DiffusionGemma深度拆解：从逐字蹦到整块喷，
// LLM生成范式的结构性跃迁", 架构解剖 2 and the encoder/decoder diagram); the canvas's
// own K/V are recomputed every step (架构解剖 2). Per query head q (KV head
// g = q / (Hq/Hk)): O = softmax(Q K^T / sqrt(h)) V over [prefix keys; canvas keys].
//
// Unit of work: two 128-query tiles ("slots" A and B) that read the same KV
// head of the same request -- the two query tiles of one head, or the same
// tile of two heads of one KV group -- walked over the request's key tiles
// (prefix tiles from the request's own tensor map, then canvas tiles). Every
// K and V tile feeds both slots' MMAs, so a tile crosses L2 -> SM once for
// 256 queries.
// Stream-K schedule: the units' key tiles form one sequence (pair-major, so
// that the units sharing a KV head run side by side) and CTA c of G walks
// tiles [c T / G, (c + 1) T / G) of it, so every CTA gets
// the same number of key tiles whatever the unit count; where its range
// crosses from one unit into the next, the CTA finishes the first unit's part
// (a segment), loads the next unit's Q and goes on. A unit walked whole by
// one CTA is normalised and stored as bf16; the parts of a unit that several
// CTAs shared go to a partial buffer (unnormalised O and the running (max,
// sum)), one slot per CTA, and attn_merge_kernel combines them.
// The walk goes through a 3-slot K ring and a 2-slot V ring:
//   warp 0   : TMA producer: Q_A and Q_B per segment (after the previous
//              segment's last QK); K tiles one ahead of V tiles
//              (a K slot frees when both slots' QK are done, a V slot when
//              both PVs are); prompt tiles a few ahead are prefetched into L2
//   warp 1   : TMEM allocator and MMA issuer. Per key tile j, in this order:
//              PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j), where QK_x(j) is
//              S_x = Q_x K_j^T (M = N = 128, K = 128) and PV_x(j) is
//              O_x += P_x V_j with P_x read from tensor memory (V as an
//              MN-major operand). tcgen05.mma ops of one thread execute in
//              issue order, so QK_x(j) may overwrite the columns PV_x(j-1)
//              reads P_x from, and the commit after QK_x(j) also covers
//              PV_x(j-1).
//   warps 2-5: softmax of slot A, warps 6-9: softmax of slot B, one query
//              row per thread: read S_x from TMEM, mask keys past the tile's
//              end, exponentiate in base 2 against a running maximum, write
//              P_x (bf16 pairs) over the first 64 columns of S_x. While one
//              slot's warps exponentiate, the tensor core runs the other
//              slot's MMAs, so the MUFU and the tensor pipe stay busy
//              together. The running maximum is raised only when the tile's
//              maximum exceeds it by more than 8 (a factor 256), and then O_x
//              and the running sum are rescaled in place; the decision is per
//              warp, since the TMEM accesses are warp-collective.
// TMEM columns: S_A [0,128) | S_B [128,256) | O_A [256,384) | O_B [384,512);
// P_x occupies columns [0,64) of S_x. A segment's first PV_x overwrites O_x;
// the softmax warps have read the previous segment's O_x before they release
// that PV (p_full).
#include <cstring>

#include "dg_internal.cuh"
#include "dg_sm100.cuh"
#include "dg_tmap.cuh"

namespace dg {
namespace attntc {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kTile = 128;
constexpr int kAtom = 128 * 128;       // 128 rows x 128 B = 16 KB
constexpr int kMatBytes = 2 * kAtom;   // a 128 x 128 bf16 tile = 32 KB
constexpr int kKSlots = 3;             // K ring depth
constexpr int kVSlots = 2;             // V ring depth
// smem: Q_A Q_B | K0 K1 K2 | V0 V1 | barriers. The dynamic shared window
// starts 1024-aligned (after the CTA's reserved 1 KB); the kernel checks this
// instead of reserving alignment slack.
constexpr int kOffQ = 0;
constexpr int kOffK = 2 * kMatBytes;
constexpr int kOffV = kOffK + kKSlots * kMatBytes;
constexpr int kOffBar = kOffV + kVSlots * kMatBytes;
constexpr int kSmemBytes = kOffBar + 256;
static_assert(kSmemBytes <= 232448, "attention tile exceeds the opt-in shared memory of a CTA");
constexpr int kMaxReq = 8;
constexpr float kRescaleThreshold = 8.f;  // log2 units
constexpr int kAhead = 4;                 // prompt-prefix tiles prefetched into L2 ahead of their load
// TMEM column of slot x's scores (and P) and of its output accumulator
__host__ __device__ constexpr uint32_t col_s(int x) { return (uint32_t)x * 128u; }
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + (uint32_t)x * 128u; }

struct Maps {
  CUtensorMap q;    // [B*C][Hq*h]
  CUtensorMap kc;   // [B*C][Hk*h]
  CUtensorMap vc;
  CUtensorMap pk[kMaxReq];  // [S_b][Hk*h] per request of this launch
  CUtensorMap pv[kMaxReq];
};

struct Params {
  int b0, nreq;  // requests [b0, b0 + nreq) in this launch
  int C, Hq, Hk;
  int S[kMaxReq];
  int q_tiles;       // 128-query tiles per canvas
  int items;         // (head, query tile) pairs per (request, KV head) = (Hq/Hk) * q_tiles
  int pairs;         // units per (request, KV head) = ceil(items / 2)
  // stream-K schedule: unit (request lb, KV head g, pair) has nt[lb] key
  // tiles; the units' tiles form one sequence of T = pairs * Tp tiles, pair
  // major (plane `pair` holds the units (lb, g) of that pair, request-major),
  // and CTA c walks tiles [c T / G, (c + 1) T / G) of it. With G a multiple of
  // `pairs`, CTAs c and c + G / pairs walk the same key tiles of the same KV
  // head at the same time (for different query tiles), so a K/V tile is read
  // from HBM once and served from L2 to the other
  int G, T, Tp;
  int nt[kMaxReq];
  int reqoff[kMaxReq];  // first tile of request lb's units within a plane
  int rows_total;    // B_total * C * Hq (partial buffer row count)
  float scale_log2;  // log2(e) / sqrt(h)
  __nv_bfloat16* O;  // [B*C][Hq*h]
  float* part_o;     // [slots][rows_total][128]
  float* part_ml;    // [slots][rows_total][2]
  int* err;
};

// First tile of CTA c's range, and the CTA whose range holds tile x.
__host__ __device__ __forceinline__ int range_lo(int c, int T, int G) { return (int)(((long long)c * T) / G); }
__host__ __device__ __forceinline__ int cta_of(int x, int T, int G) {
  return (int)(((long long)(x + 1) * G + T - 1) / T) - 1;
}

// One unit's share of a CTA's range: request lb, KV head g, pair, key tiles
// [j0, j1) of the unit's nt, and where the unit's partial results go: parts
// CTAs share the unit and this one writes slot `slot` (parts == 1: the
// normalised output directly).
struct Segment {
  int lb, g, pair, j0, j1, nt, parts, slot;
};

// The segment of CTA c that starts at tile x of the sequence (x inside c's
// range [x, hi)).
__device__ __forceinline__ Segment segment_at(const Params& p, int x, int hi, int c) {
  Segment sg;
  const int pl = x / p.Tp;  // pair plane
  const int x0 = x - pl * p.Tp;
  int lb = 0;
  while (lb + 1 < p.nreq && p.reqoff[lb + 1] <= x0) ++lb;
  const int nt = p.nt[lb];
  const int rel = x0 - p.reqoff[lb];
  const int g = rel / nt;
  const int uoff = pl * p.Tp + p.reqoff[lb] + g * nt;
  sg.lb = lb;
  sg.g = g;
  sg.pair = pl;
  sg.nt = nt;
  sg.j0 = rel - g * nt;
  sg.j1 = min(hi, uoff + nt) - uoff;
  const int first = cta_of(uoff, p.T, p.G);
  sg.parts = cta_of(uoff + nt - 1, p.T, p.G) - first + 1;
  sg.slot = c - first;
  return sg;
}

__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk) {
  // K-major 128-row operand with 128 columns of K split into two 64-wide atoms
  return umma_desc_sw128(base + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024);
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ Maps maps, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // SW128 tiles need 1024-byte alignment (uniform: no TMEM held yet)
    if (threadIdx.x == 0) set_error(p.err, kDevBadAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bar + 0;                   // [2] Q_x landed
  uint64_t* q_empty = bar + 2;                  // [2] the segment's last QK_x done (Q_x may be replaced)
  uint64_t* k_full = bar + 4;                   // [3]
  uint64_t* k_empty = k_full + kKSlots;         // [3] the last slot's QK of the tile done
  uint64_t* v_full = k_empty + kKSlots;         // [2]
  uint64_t* v_empty = v_full + kVSlots;         // [2] the last slot's PV of the tile done
  uint64_t* s_full = v_empty + kVSlots;         // [2] S_x in TMEM (and PV_x of the previous tile done)
  uint64_t* p_full = s_full + 2;                // [2] P_x in TMEM (4 warps)
  uint64_t* pv_done = p_full + 2;               // [2] every MMA of slot x in the segment done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(pv_done + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int lo = range_lo(cta, p.T, p.G), hi = range_lo(cta + 1, p.T, p.G);
  // the segments of [lo, hi): every role walks the same list
  auto nslots_of = [&](const Segment& sg) { return min(2, p.items - 2 * sg.pair); };
  // (query head, query tile) of slot x; slot B repeats A's when it is unused
  auto slot_head = [&](const Segment& sg, int x) {
    return sg.g * (p.Hq / p.Hk) + min(2 * sg.pair + x, p.items - 1) / p.q_tiles;
  };
  auto slot_tile = [&](const Segment& sg, int x) { return min(2 * sg.pair + x, p.items - 1) % p.q_tiles; };
  auto nps_of = [&](const Segment& sg) { return (p.S[sg.lb] + kTile - 1) / kTile; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  griddep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n = hi - lo;  // key tiles of this CTA, over all its segments

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      // flat tile i of this CTA (tile lo + i of the sequence): K and V rows
      // [y, y + 128) of its request's prompt prefix or canvas, KV head g
      auto tile_src = [&](int i, const CUtensorMap*& mk, const CUtensorMap*& mv, int& y, int& g, bool& prompt) {
        const Segment sg = segment_at(p, lo + i, hi, cta);
        const int nps = nps_of(sg);
        const int j = sg.j0;  // segment_at starts the segment at this tile
        g = sg.g;
        prompt = j < nps;
        if (prompt) {
          mk = &maps.pk[sg.lb];
          mv = &maps.pv[sg.lb];
          y = j * kTile;
        } else {
          mk = &maps.kc;
          mv = &maps.vc;
          y = (p.b0 + sg.lb) * p.C + (j - nps) * kTile;
        }
      };
      auto load_k = [&](int i) {
        const CUtensorMap *mk, *mv;
        int y, g;
        bool pr;
        tile_src(i, mk, mv, y, g, pr);
        mbar_arrive_expect_tx(&k_full[i % kKSlots], kMatBytes);
        tma_load_3d(smem + kOffK + (i % kKSlots) * kMatBytes, mk, &k_full[i % kKSlots], 0, y, g * 2, pol);
      };
      auto load_v = [&](int i) {
        const CUtensorMap *mk, *mv;
        int y, g;
        bool pr;
        tile_src(i, mk, mv, y, g, pr);
        mbar_arrive_expect_tx(&v_full[i % kVSlots], kMatBytes);
        tma_load_3d(smem + kOffV + (i % kVSlots) * kMatBytes, mv, &v_full[i % kVSlots], 0, y, g * 2, pol);
      };
      auto is_prompt = [&](int i) {
        const Segment sg = segment_at(p, lo + i, hi, cta);
        return sg.j0 < nps_of(sg);
      };
      // prompt-prefix tiles further ahead are pulled into L2 early
      auto prefetch = [&](int i) {
        if (i < n) {
          const Segment sg = segment_at(p, lo + i, hi, cta);
          if (sg.j0 < nps_of(sg)) {
            tma_prefetch_3d(&maps.pk[sg.lb], 0, sg.j0 * kTile, sg.g * 2);
            tma_prefetch_3d(&maps.pv[sg.lb], 0, sg.j0 * kTile, sg.g * 2);
          }
        }
      };
      // Q of segment `sg` (its active slots); qc[x] counts the segments in
      // which slot x was active, and Q_x is replaced only after the last QK_x
      // of the previous one
      uint32_t qc[2] = {0u, 0u};
      auto load_q = [&](const Segment& sg) -> bool {
        for (int x = 0; x < nslots_of(sg); ++x) {
          if (qc[x] > 0 && !mbar_wait(&q_empty[x], (qc[x] - 1) & 1, p.err, abort_flag)) return false;
          mbar_arrive_expect_tx(&q_full[x], kMatBytes);
          tma_load_3d(smem + kOffQ + x * kMatBytes, &maps.q, &q_full[x], 0,
                      (p.b0 + sg.lb) * p.C + slot_tile(sg, x) * kTile, slot_head(sg, x) * 2, pol);
          ++qc[x];
        }
        return true;
      };
      int nk = 0, nv = 0;  // next K tile and next V tile to load (flat)
      // the prompt prefix is an input of the step: its first tiles may be
      // fetched before the predecessor kernels are done
      while (nk < kKSlots && nk < n && is_prompt(nk)) load_k(nk++);
      while (nv < kVSlots && nv < n && is_prompt(nv)) load_v(nv++);
      for (int i = nk; i < nk + kAhead; ++i) prefetch(i);
      griddep_wait();
      int next_seg = lo;  // first tile of the next segment whose Q is not loaded yet
      bool ok = true;
      {
        const Segment sg = segment_at(p, lo, hi, cta);
        ok = load_q(sg);
        next_seg = lo + (sg.j1 - sg.j0);
      }
      // K runs one tile ahead of V (the MMA order is PV(j-1) then QK(j)); a
      // segment's Q is loaded just before its first K tile
      while (ok && nv < n && !*abort_flag) {
        if (nk < n && nk <= nv + 1) {
          if (lo + nk == next_seg) {
            const Segment sg = segment_at(p, next_seg, hi, cta);
            if (!(ok = load_q(sg))) break;
            next_seg += sg.j1 - sg.j0;
          }
          if (nk >= kKSlots &&
              !mbar_wait(&k_empty[nk % kKSlots], ((nk / kKSlots) - 1) & 1, p.err, abort_flag))
            break;
          load_k(nk);
          prefetch(nk + kAhead);
          ++nk;
        } else {
          if (nv >= kVSlots &&
              !mbar_wait(&v_empty[nv % kVSlots], ((nv / kVSlots) - 1) & 1, p.err, abort_flag))
            break;
          load_v(nv);
          ++nv;
        }
      }
      if (*abort_flag || !ok) {  // drain this CTA's own copies: the last Q of each slot and of each ring slot
        for (int x = 0; x < 2; ++x)
          if (qc[x] > 0) mbar_wait(&q_full[x], (qc[x] - 1) & 1, p.err, nullptr);
        for (int i = nk - kKSlots; i < nk; ++i)
          if (i >= 0) mbar_wait(&k_full[i % kKSlots], (i / kKSlots) & 1, p.err, nullptr);
        for (int i = nv - kVSlots; i < nv; ++i)
          if (i >= 0) mbar_wait(&v_full[i % kVSlots], (i / kVSlots) & 1, p.err, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, 128, false);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, true);
      bool ok = true;
      uint32_t qc[2] = {0u, 0u};  // segments in which slot x was active
      uint32_t tc[2] = {0u, 0u};  // tiles slot x has gone through (p_full phases)
      // flat tile f of this CTA; t = its index within the segment, nt_seg the
      // segment's tile count, ns its active slots
      auto qk = [&](int x, int f, int t, int nt_seg, int ns) -> bool {
        const int slot = f % kKSlots;
        if (x == 0 && !mbar_wait(&k_full[slot], (f / kKSlots) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t qbase = smem_u32(smem + kOffQ + x * kMatBytes);
        const uint32_t kbase = smem_u32(smem + kOffK + slot * kMatBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + col_s(x), kdesc(qbase, kk), kdesc(kbase, kk), id_qk, kk != 0);
        mma_commit(&s_full[x]);
        if (x == ns - 1) mma_commit(&k_empty[slot]);
        if (t == nt_seg - 1) mma_commit(&q_empty[x]);  // Q_x is not read again in this segment
        return true;
      };
      auto pv = [&](int x, int f, int t, int ns) -> bool {
        const int slot = f % kVSlots;
        if (!mbar_wait(&p_full[x], tc[x] & 1, p.err, abort_flag)) return false;
        ++tc[x];
        if (x == 0 && !mbar_wait(&v_full[slot], (f / kVSlots) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(smem + kOffV + slot * kMatBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + col_o(x), tmem + col_s(x) + kk * 8, umma_desc_sw128(vbase + kk * 2048, kAtom, 1024),
                      id_pv, (t | kk) != 0);
        if (x == ns - 1) mma_commit(&v_empty[slot]);
        return true;
      };
      for (int x0 = lo; ok && x0 < hi;) {
        const Segment sg = segment_at(p, x0, hi, cta);
        const int ns = nslots_of(sg);
        const int nt_seg = sg.j1 - sg.j0;
        const int f0 = x0 - lo;
        for (int x = 0; ok && x < ns; ++x) ok = mbar_wait(&q_full[x], qc[x] & 1, p.err, abort_flag);
        for (int x = 0; ok && x < ns; ++x) ok = qk(x, f0, 0, nt_seg, ns);
        for (int t = 0; ok && t < nt_seg; ++t) {
          for (int x = 0; ok && x < ns; ++x) {
            ok = pv(x, f0 + t, t, ns);
            if (ok && t + 1 < nt_seg) ok = qk(x, f0 + t + 1, t + 1, nt_seg, ns);
          }
        }
        // every MMA of the segment has landed in O before the softmax warps
        // read it
        for (int x = 0; x < ns; ++x) {
          mma_commit(&pv_done[x]);
          ++qc[x];
        }
        x0 += nt_seg;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int x = (warp - 2) >> 2;  // slot of this warpgroup
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_col = col_s(x), o_col = col_o(x);
    uint32_t tc = 0, qc = 0;  // tiles and segments this slot has gone through
    bool ok = true;
    for (int x0 = lo; ok && x0 < hi;) {
      // only what the tile loop needs stays live across it; the segment is
      // looked up again for the output
      const int xs = x0;
      int nt_seg, j0, nps, S;
      {
        const Segment sg = segment_at(p, x0, hi, cta);
        nt_seg = sg.j1 - sg.j0;
        x0 += nt_seg;
        if (x >= nslots_of(sg)) continue;  // slot unused in this segment
        j0 = sg.j0;
        nps = nps_of(sg);
        S = p.S[sg.lb];
      }
      float m_run = -INFINITY, l = 0.f;
      for (int i = 0; ok && i < nt_seg; ++i, ++tc) {
        if (!(ok = mbar_wait_warp(&s_full[x], tc & 1, p.err, abort_flag))) break;
        tc_fence_after();
        float v[128];
        {
          uint32_t u[128];
          tmem_ld128_sync(tmem + lane_off + s_col, u);
#pragma unroll
          for (int e = 0; e < 128; ++e) v[e] = __uint_as_float(u[e]);
        }
        // keys of this tile that exist
        const int j = j0 + i;
        const int valid = (j < nps) ? min(kTile, S - j * kTile) : min(kTile, p.C - (j - nps) * kTile);
        if (valid < kTile) {  // ragged last tile (uniform over the CTA)
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) v[c] = -INFINITY;
        }
        // row maximum: 8 independent chains of three-input maxima over 16
        // scores each, then a tree over the chains
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float* w = v + 16 * k;
          float a = fmax3(w[0], w[1], w[2]);
#pragma unroll
          for (int c = 3; c < 15; c += 2) a = fmax3(a, w[c], w[c + 1]);
          mx[k] = fmaxf(a, w[15]);
        }
        const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                         p.scale_log2;  // the scale is positive: maximum of the scaled scores
        // The O rows live in TMEM and are rescaled with warp-collective
        // tcgen05.ld/st, so the decision is taken per warp: when any row of the
        // warp has outgrown its maximum by the threshold, every row of the warp
        // moves its maximum up to its tile maximum (alpha = 1 where it stays).
        const bool rescale = __any_sync(0xffffffffu, mt > m_run + kRescaleThreshold);
        float alpha = 1.f;
        if (rescale) {
          const float m_new = fmaxf(m_run, mt);
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(s scale - m_run) as bf16 pairs, row sum over 8 chains
        uint32_t pk[64];
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float neg_m = -m_run;
        // full tiles and the ragged last tile run separate copies of this loop:
        // compiled apart, neither spills registers (as one loop, 144 bytes did)
        if (valid == kTile) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float p0 = ex2_approx(fmaf(v[2 * c], p.scale_log2, neg_m));
            const float p1 = ex2_approx(fmaf(v[2 * c + 1], p.scale_log2, neg_m));
            ls[(2 * c) & 7] += p0;
            ls[(2 * c + 1) & 7] += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[c] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float p0 = ex2_approx(fmaf(v[2 * c], p.scale_log2, neg_m));
            const float p1 = ex2_approx(fmaf(v[2 * c + 1], p.scale_log2, neg_m));
            ls[(2 * c) & 7] += p0;
            ls[(2 * c + 1) & 7] += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[c] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        }
        // s_full(i) was committed after PV_x(i-1): O_x holds it and may be rescaled
        if (rescale && i > 0) {
          l *= alpha;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tmem_ld32_sync(tmem + lane_off + o_col + c * 32, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(tmem + lane_off + o_col + c * 32, u);
          }
        }
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        {
          uint32_t u[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = pk[e];
          tmem_st32(tmem + lane_off + s_col, u);
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = pk[32 + e];
          tmem_st32(tmem + lane_off + s_col + 32, u);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      if (!mbar_wait_warp(&pv_done[x], qc & 1, p.err, abort_flag)) {
        ok = false;
        break;
      }
      ++qc;
      tc_fence_after();
      const Segment sg = segment_at(p, xs, hi, cta);
      const int qrow = slot_tile(sg, x) * kTile + r;
      const bool has_row = qrow < p.C;
      const size_t grow = (size_t)((p.b0 + sg.lb) * p.C + qrow);
      const float inv = 1.f / l;
      const int q = slot_head(sg, x);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t u[32];
        tmem_ld32_sync(tmem + lane_off + o_col + cc * 32, u);
        if (!has_row) continue;
        if (sg.parts == 1) {  // the whole unit ran here: normalised output
          uint4* dst = reinterpret_cast<uint4*>(p.O + grow * p.Hq * 128 + q * 128 + cc * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            __nv_bfloat162* w2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w2[e] = __floats2bfloat162_rn(__uint_as_float(u[v4 * 8 + 2 * e]) * inv,
                                            __uint_as_float(u[v4 * 8 + 2 * e + 1]) * inv);
            dst[v4] = w;
          }
        } else {  // one of the unit's parts: unnormalised O and (max, sum)
          const size_t prow_i = (size_t)sg.slot * p.rows_total + grow * p.Hq + q;
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow_i * 128 + cc * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(u[4 * v4]), __uint_as_float(u[4 * v4 + 1]),
                                  __uint_as_float(u[4 * v4 + 2]), __uint_as_float(u[4 * v4 + 3]));
          if (cc == 0) {
            p.part_ml[prow_i * 2] = m_run;
            p.part_ml[prow_i * 2 + 1] = l;
          }
        }
      }
      // the O reads are complete (tmem_ld32_sync waits) before this warp's
      // next p_full arrival lets the next segment's first PV overwrite O
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Combine the parts of the units that several CTAs shared: m = max m_z,
// w_z = 2^(m_z - m), O = sum_z w_z O_z / sum_z w_z l_z (parts in slot order).
// One warp per (row, head) of this launch's requests, 4 dims per lane, so
// the merge of every shared unit is spread over the whole GPU with coalesced
// loads; rows whose unit ran whole in one CTA were written by it and are
// skipped.
__global__ void attn_merge_kernel(Params p) {
  griddep_launch();
  griddep_wait();
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= p.nreq * p.C * p.Hq) return;
  const int lb = w / (p.C * p.Hq);
  const int qrow = (w / p.Hq) % p.C;
  const int q = w % p.Hq;
  const int grp = p.Hq / p.Hk;
  const int item = (q % grp) * p.q_tiles + qrow / kTile;
  const int nt = p.nt[lb];
  const int uoff = (item / 2) * p.Tp + p.reqoff[lb] + (q / grp) * nt;
  const int parts = cta_of(uoff + nt - 1, p.T, p.G) - cta_of(uoff, p.T, p.G) + 1;
  if (parts == 1) return;
  const size_t row = (size_t)p.b0 * p.C * p.Hq + w;
  float m = -INFINITY;
  for (int z = 0; z < parts; ++z) m = fmaxf(m, p.part_ml[((size_t)z * p.rows_total + row) * 2]);
  float l = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
  for (int z = 0; z < parts; ++z) {
    const size_t rz = (size_t)z * p.rows_total + row;
    const float wz = ex2_approx(p.part_ml[rz * 2] - m);
    l += wz * p.part_ml[rz * 2 + 1];
    const float4 v = reinterpret_cast<const float4*>(p.part_o + rz * 128)[lane];
    o0 += wz * v.x;
    o1 += wz * v.y;
    o2 += wz * v.z;
    o3 += wz * v.w;
  }
  const float inv = 1.f / l;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(p.O + row * 128 + lane * 4);
  dst[0] = __floats2bfloat162_rn(o0 * inv, o1 * inv);
  dst[1] = __floats2bfloat162_rn(o2 * inv, o3 * inv);
}

// Units (request, KV head, pair of (head, query tile)) per request.
int attn_units_per_request(int C, int Hq, int Hk) {
  const int items = (Hq / Hk) * ceil_div(C, kTile);
  return Hk * ceil_div(items, 2);
}

}  // namespace attntc

// ---------------------------------------------------------------- host side
// Schedule of one launch (requests S[0..nreq)): the units' key tiles in one
// sequence of T tiles over G CTAs. When every unit can take the same number
// s of CTAs and U * s CTAs fill at least 90 % of the SMs, G = U * s: with
// equal unit lengths the CTA ranges then split each unit evenly and no range
// crosses a unit boundary (one Q load and one output pass per CTA). Otherwise
// (e.g. 64 units on 148 SMs, where the even split would leave 20 idle) G is
// the SM count and ranges cross units (stream-K). Either way no unit is shared
// by more than parts_cap CTAs (the partial buffers hold that many parts per
// row): G shrinks until that holds.
static AttnTc::Sched attn_sched(int nreq, const int* S, int C, int Hq, int Hk, int sm_count, int parts_cap) {
  AttnTc::Sched sc;
  const int pairs = ceil_div((Hq / Hk) * ceil_div(C, attntc::kTile), 2);
  const int U = pairs * Hk * nreq;
  sc.Tp = 0;
  int nt_min = 1 << 30;
  for (int lb = 0; lb < nreq; ++lb) {
    sc.nt[lb] = ceil_div(S[lb], attntc::kTile) + ceil_div(C, attntc::kTile);
    sc.reqoff[lb] = sc.Tp;
    sc.Tp += Hk * sc.nt[lb];
    nt_min = std::min(nt_min, sc.nt[lb]);
  }
  sc.T = pairs * sc.Tp;
  auto parts_max = [&](int G) {
    int mx = 1;
    for (int pl = 0; pl < pairs; ++pl)
      for (int lb = 0; lb < nreq; ++lb)
        for (int g = 0; g < Hk; ++g) {
          const int off = pl * sc.Tp + sc.reqoff[lb] + g * sc.nt[lb];
          mx = std::max(mx, attntc::cta_of(off + sc.nt[lb] - 1, sc.T, G) - attntc::cta_of(off, sc.T, G) + 1);
        }
    return mx;
  };
  const int s_even = std::max(1, std::min(sm_count / std::max(1, U), nt_min));
  int G = (10 * U * s_even >= 9 * sm_count) ? U * s_even : sm_count - sm_count % pairs;
  G = std::max(1, std::min(G, sc.T));
  while (G > 1 && parts_max(G) > parts_cap) --G;
  sc.G = G;
  sc.parts = parts_max(G);
  return sc;
}

int attn_tc_slots(int B, int C, int Hq, int Hk, const int* S, int sm_count) {
  int slots = 1;
  for (int b0 = 0; b0 < B; b0 += attntc::kMaxReq)
    slots = std::max(slots, attn_sched(std::min(attntc::kMaxReq, B - b0), S + b0, C, Hq, Hk, sm_count, 1 << 20).parts);
  return slots;
}

bool attn_tc_prepare(AttnTc* at, const AttnShape& sh, const void* Q, const void* Kc, const void* Vc,
                     const int32_t* S, const void* const* pk, const void* const* pv, void* O, float* part_o,
                     float* part_ml, int slots, int sm_count) {
  if (cudaFuncSetAttribute(attntc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           attntc::kSmemBytes) != cudaSuccess) {
    set_last_error("cudaFuncSetAttribute(attn_tc_kernel) failed");
    return false;
  }
  if (sh.h != 128) {
    set_last_error("attn_tc: head_dim must be 128");
    return false;
  }
  at->sh = sh;
  at->O = O;
  at->part_o = part_o;
  at->part_ml = part_ml;
  at->groups.clear();
  // [rows][heads * 128] bf16 as 3D (64 elements, rows, heads * 2): one box
  // (64, 128, 2) is a head's 128 x 128 tile as two 128-byte-swizzled halves
  const uint64_t rows = (uint64_t)sh.B * sh.C;
  const uint64_t dq[3] = {64, rows, (uint64_t)sh.Hq * 2}, sq[2] = {(uint64_t)sh.Hq * 256, 128};
  const uint64_t dk[3] = {64, rows, (uint64_t)sh.Hk * 2}, sk[2] = {(uint64_t)sh.Hk * 256, 128};
  const uint32_t box[3] = {64, 128, 2};
  for (int b0 = 0; b0 < sh.B; b0 += attntc::kMaxReq) {
    AttnTc::Group grp;
    grp.b0 = b0;
    grp.nreq = std::min(attntc::kMaxReq, sh.B - b0);
    grp.sched = attn_sched(grp.nreq, S + b0, sh.C, sh.Hq, sh.Hk, sm_count, part_o ? slots : 1);
    static_assert(sizeof(attntc::Maps) <= sizeof(grp.maps), "AttnTc map storage too small");
    attntc::Maps* m = reinterpret_cast<attntc::Maps*>(grp.maps);
    memset(grp.maps, 0, sizeof(grp.maps));
    if (!encode_tmap_bf16(&m->q, Q, 3, dq, sq, box, true) || !encode_tmap_bf16(&m->kc, Kc, 3, dk, sk, box, true) ||
        !encode_tmap_bf16(&m->vc, Vc, 3, dk, sk, box, true))
      return false;
    for (int i = 0; i < grp.nreq; ++i) {
      const int b = b0 + i;
      grp.S[i] = S[b];
      if (S[b] > 0) {
        const uint64_t dp[3] = {64, (uint64_t)S[b], (uint64_t)sh.Hk * 2};
        if (!encode_tmap_bf16(&m->pk[i], pk[b], 3, dp, sk, box, true) ||
            !encode_tmap_bf16(&m->pv[i], pv[b], 3, dp, sk, box, true))
          return false;
      }
    }
    at->groups.push_back(grp);
  }
  return true;
}

void launch_attn_tc(Exec& ex, const AttnTc& at) {
  const AttnShape& sh = at.sh;
  const int q_tiles = ceil_div(sh.C, 128);
  const int rows_total = sh.B * sh.C * sh.Hq;
  const int items = (sh.Hq / sh.Hk) * q_tiles;
  for (const auto& grp : at.groups) {
    attntc::Params p;
    p.b0 = grp.b0;
    p.nreq = grp.nreq;
    p.C = sh.C;
    p.Hq = sh.Hq;
    p.Hk = sh.Hk;
    for (int i = 0; i < attntc::kMaxReq; ++i) {
      p.S[i] = i < grp.nreq ? grp.S[i] : 0;
      p.nt[i] = i < grp.nreq ? grp.sched.nt[i] : 1;
      p.reqoff[i] = i < grp.nreq ? grp.sched.reqoff[i] : grp.sched.Tp;
    }
    p.q_tiles = q_tiles;
    p.items = items;
    p.pairs = ceil_div(items, 2);
    p.G = grp.sched.G;
    p.T = grp.sched.T;
    p.Tp = grp.sched.Tp;
    p.rows_total = rows_total;
    p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
    p.O = static_cast<__nv_bfloat16*>(at.O);
    p.part_o = at.part_o;
    p.part_ml = at.part_ml;
    p.err = ex.err;
    launch_pdl(attntc::attn_tc_kernel, dim3(p.G), dim3(attntc::kThreads), attntc::kSmemBytes, ex.stream,
               *reinterpret_cast<const attntc::Maps*>(grp.maps), p);
    ex.launches++;
    if (grp.sched.parts > 1) {
      launch_pdl(attntc::attn_merge_kernel, dim3(ceil_div(grp.nreq * sh.C * sh.Hq, 8)), dim3(256), 0, ex.stream,
                 p);
      ex.launches++;
    }
  }
}

}  // namespace dg
