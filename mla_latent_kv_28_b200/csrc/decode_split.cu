// Split-KV decode attention over the latent cache on the sm_100a tensor core.
//
// Per (sequence, split) segment, for all 128 heads at once (heads are the MMA's M = 128):
//   S = Q_abs [128 x 576] . [c ; k^R]^T [576 x 64 tokens]     (tcgen05, fp32 in TMEM)
//   online softmax over the tokens (exp2, running max with lazy rescale)
//   O += P [128 x 64] . c [64 x 512]                            (tcgen05, fp32 in TMEM)
// and the segment's partial O / l and log-sum-exp go to the split slots.
//
// Why a 2-CTA cluster: O alone (128 heads x 512 fp32) is the whole 256 KB of one SM's
// tensor memory, leaving no room for S. So the two CTAs of a cluster split the 576 columns
// of every cache row: CTA r holds c^KV columns [256r, 256r+256) and k^R columns
// [32r, 32r+32) (288 columns), computes the partial scores over them, and keeps the O
// columns [256r, 256r+256). The partial score tiles cross between the two CTAs through
// distributed shared memory (one bulk copy per warp, 16-bit block floating point); each CTA
// adds its own exact partial to the peer's. Each cache byte is read from HBM once, by one CTA.
//
// Pipeline (64-token tiles, g = tile index within this cluster's work):
//   TMA ring of 4 stages -> QK(g) into S -> softmax warpgroup g % 2: S out of TMEM, partial
//   to the peer and the peer's back, max, exponentials, P(g) -> PV(g) into O.
// Two softmax warpgroups take alternate tiles, so each has two tile periods for one tile.
// QK and PV have issuer warps of their own (one thread issues an MMA only every ~60-90
// cycles).
// Segment boundaries (a unit may hold the tail of one sequence and the head of the next)
// are handled by a separate warpgroup: it loads the next segment's query columns as soon as
// the last QK of the previous segment is done, and writes the finished segment's O / l
// while the next segment is already running.
//
// Tensor memory (512 columns per CTA): O [0,256) fp32, S [256,320) fp32, P [320,384) bf16x2
// (one 32-column P per softmax warpgroup), Q [384,512) bf16x2 (the CTA's 256 c^KV query
// columns, the A operand of the QK MMAs). The CTA's 32 k^R query columns are the A operand of
// the two k^R MMAs from shared memory.
// Shared memory: 4 stages x 36 KB of cache tiles (four 64x64 c^KV boxes with 128-byte
// swizzle + one 64x32 k^R box with 64-byte swizzle), 4 x 16.5 KB exchange buffers, the 8 KB
// k^R query operand, per-segment (max, sum), mbarriers.
// Warps: 0 TMA producer, 1 QK issuer (and TMEM owner), 2 PV issuer, 3 idle; 4..7 and 8..11
// the two softmax warpgroups, one thread per head (= TMEM lane) and all 64 tokens of a tile;
// 12..15 segment transitions (query load, epilogue).
//
// A quantised cache (E4M3 codes, one power-of-two scale per row) runs through a second
// instantiation: the producer lands each tile's codes in the upper halves of the stage's bf16
// boxes, the transition warpgroup expands them in place to exactly the bf16 rows (see
// e4m3_expand.cuh) and only then lets the tile's QK go; the rest is the same kernel.
//
// Every wait is bounded: after about a second it sets the device error word (timeout bit)
// and the CTA's abort flag, all roles leave their loops, wait for their own copies and
// MMAs in flight, and the CTA frees its tensor memory and exits.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "e4m3_bf16.cuh"
#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kT = 64;                    // tokens per tile (the plan's tile)
constexpr int kStages = 4;
constexpr int kKSteps = 18;               // 288 columns / 16
constexpr uint32_t kBoxC = kT * 128;      // 8 KB: 64 tokens x 64 c^KV columns
constexpr uint32_t kBoxR = kT * 64;       // 4 KB: 64 tokens x 32 k^R columns
constexpr uint32_t kStageBytes = 4 * kBoxC + kBoxR;   // 36 KB
// Partial scores cross between the two CTAs as 16-bit block floating point: per (head, tile)
// 64 integers and one power-of-two scale. A softmax warp's block: 32 rows (heads) of 128 bytes,
// then the 32 scale exponents. Each softmax warpgroup has two buffers of 4 blocks.
constexpr uint32_t kXBlockBytes = 32 * 128 + 32 * 4;   // 4224
constexpr uint32_t kXBufBytes = 4 * kXBlockBytes;       // one tile of one warpgroup (16.5 KB)
constexpr uint32_t kOffXin = kStages * kStageBytes;
constexpr uint32_t kOffQr = kOffXin + 4 * kXBufBytes;  // [128 heads][32 k^R query columns], 64-byte swizzle
constexpr uint32_t kQrBytes = 128 * 64;                 // 8 KB: the A operand of the two k^R MMAs
constexpr uint32_t kOffMl = kOffQr + kQrBytes;         // [2 segs][2 warpgroups][128] float2 (max, sum)
constexpr uint32_t kOffMh = kOffMl + 2 * 2 * 128 * 8;  // [128] float: running max handed between warpgroups
constexpr uint32_t kOffEpi = kOffMh + 128 * 4;      // [128] int: segments whose epilogue read head h's (max, sum)
constexpr uint32_t kOffBars = kOffEpi + 128 * 4;

// barrier indices
constexpr int kBarKvFull = 0;                    // [kStages] TMA landed
constexpr int kBarKvEmpty = kStages;             // [kStages] PV of the tile done
// The softmax warpgroups take alternate tiles, so the signals between them and the issuers come
// in pairs indexed by tile parity: each waiter then steps through the consecutive phases of
// its own barrier, and a phase parity never names two different tiles.
constexpr int kBarSFull = 2 * kStages;           // [2] partial S of tile g in TMEM (g % 2)
constexpr int kBarSEmpty = kBarSFull + 2;        // [2] the softmax copied S(g) out
constexpr int kBarPFull = kBarSFull + 4;         // [2] P(g) in TMEM, O rescaled, V tail zeroed
constexpr int kBarPvDone = kBarSFull + 6;        // [4] PV(g) finished (g % 4: see the softmax's waits)
constexpr int kBarQReady = kBarSFull + 11;       // query columns of the next segment in TMEM
constexpr int kBarQFree = kBarSFull + 12;        // the last QK of a segment finished
constexpr int kBarOFull = kBarSFull + 13;        // the last PV of a segment finished
constexpr int kBarOFree = kBarSFull + 14;        // the epilogue has read O
constexpr int kBarMlFull = kBarSFull + 15;       // (max, sum) of a finished even segment in smem
constexpr int kBarFinal = kBarSFull + 16;        // all MMAs of this CTA done (teardown)
constexpr int kBarFinal2 = kBarSFull + 17;       // all PV MMAs done (teardown)
constexpr int kBarXFull = kBarSFull + 18;        // [2 warpgroups][2 buffers][4 warps] peer's block landed
constexpr int kBarQReady0 = kBarXFull + 16;      // the first segment's query columns in TMEM
constexpr int kBarQLanded = kBarQReady0 + 1;     // ... and in shared memory (stages 1-2)
constexpr int kBarMHand = kBarQLanded + 1;       // [4 head quarters] running max of tile g-1 published
constexpr int kBarMlFull1 = kBarMHand + 4;      // ... of a finished odd segment
constexpr int kBarKvConv = kBarMlFull1 + 1;     // [kStages] quantised cache: the tile expanded to bf16
constexpr int kBarConvSync = kBarKvConv + kStages;   // quantised cache: the expanding warpgroup's codes are read
constexpr int kNumBars = kBarConvSync + 1;
// The first segment's query columns arrive by TMA in stages 1-2 (exactly 72 KB: four 64-column
// boxes of 128 heads with 128-byte swizzle, then one 32-column k^R box with 64-byte swizzle);
// the producer fills those stages with cache tiles only after the query has moved to TMEM.
constexpr uint32_t kQBoxC = 128 * 128;   // 16 KB
constexpr uint32_t kQBytes = 4 * kQBoxC + 128 * 64;
static_assert(kQBytes == 2 * kStageBytes, "query staging fills stages 1-2 exactly");
constexpr uint32_t kOffMisc = kOffBars + 8 * kNumBars;
constexpr uint32_t kSmemUsed = kOffMisc + 128;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;     // room to align the base to 1 KB
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");

// Tensor memory: O, S, one P per softmax warpgroup (tile parity), the c^KV query columns.
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemP = 320, kTmemQ = 384, kTmemCols = 512;
static_assert(kTmemS + kT <= kTmemP && kTmemP + 2 * (kT / 2) <= kTmemQ && kTmemQ + 128 <= kTmemCols, "TMEM map");
static_assert(kOffQr % 1024 == 0, "swizzled operand alignment");
constexpr int kThreads = 512;   // 16 warps = 4 warpgroups (roles below)
// Register split between the warpgroups (setmaxnreg), against 512 x 128 at launch:
// 128 x (88 + 160 + 160 + 96) = 64,512 <= 65,536.
constexpr int kRegsLaunch = 128, kRegsCtrl = 88, kRegsSoftmax = 160, kRegsTrans = 96;
static_assert(128 * (kRegsCtrl + 2 * kRegsSoftmax + kRegsTrans) <= kThreads * kRegsLaunch, "register split");
static_assert(kBarPvDone + 4 <= kBarSFull + 11, "barrier map");
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kT, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);
constexpr float kRescaleThreshold = 8.f;   // log2 units: rescale O only when the max grows more

struct Params {
  const __nv_bfloat16* q_abs;
  PlanView plan;
  int batch, n_heads;      // n_heads: attention rows per sequence, token-major (heads x new tokens)
  int q_len, heads_per_token;   // new tokens per sequence; row r is token r / heads_per_token
  int row_base, q_row_stride;   // this launch's rows: [row_base, row_base + n_heads) of q_row_stride
  int64_t seq_stride;
  const int32_t* page_table;
  int max_pages, num_pages;
  float scale_log2;
  float* part_o;
  float* part_lse;
  uint32_t* err;
  long long wait_limit;
  // quantised cache (E4M3 codes + one power-of-two scale per row), else kv_exp == nullptr
  const int8_t* kv_exp;
  int64_t kv_rows;          // rows of the cache, for the bounds of the exponent loads
  // prefill (the kPrefill instantiation): a work item is one head and 128 consecutive new
  // tokens of one sequence, taken whole by one cluster, whose latent rows go to the output
  int q_tokens;             // T, new tokens per sequence
  int n_blocks;             // 128-token blocks per head: ceil(T / 128)
  int n_items;              // batch * heads * n_blocks
  const int32_t* kv_lens;
  int64_t max_kv_len;
  __nv_bfloat16* out_latent;   // [B, T, n_h, 512]
  float* out_lse;              // [B, T, n_h] or nullptr
};

// Walks this cluster's work tile by tile: units in turn, the segments (one sequence's
// tokens inside a unit) of each unit, and the 32-token tiles of each segment.
struct TileCursor {
  int u, b, ub, ue;        // unit, sequence, the unit's plan-tile range
  int slot, len, j0, j1;   // the segment: partial slot, kv_len, token range [j0, j1)
  int k, nk;               // tile within the segment, tiles in the segment
  uint32_t g, seg;         // tile and segment counters of this cluster
  bool valid;

  __device__ __forceinline__ bool enter_sequence(const Params& p) {
    // find the next sequence of the current unit that overlaps it; false if none
    for (; b < p.batch && p.plan.seq_tile[b] < ue; ++b) {
      const int tb = p.plan.seq_tile[b], te = p.plan.seq_tile[b + 1];
      if (te <= ub) continue;
      len = p.plan.seq_len[b];
      j0 = (max(ub, tb) - tb) * kTileTokens;
      j1 = min((min(ue, te) - tb) * kTileTokens, len);
      nk = (j1 - j0 + kT - 1) / kT;
      slot = p.plan.seq_slot[b] + (u - p.plan.seq_unit[b]);
      k = 0;
      return true;
    }
    return false;
  }
  __device__ __forceinline__ void find(const Params& p) {
    const int n_units = p.plan.header[1];
    for (; u < n_units; u += (int)num_clusters_x()) {
      ub = p.plan.unit_begin[u];
      ue = p.plan.unit_begin[u + 1];
      if (enter_sequence(p)) { valid = true; return; }
      b = u + (int)num_clusters_x() < n_units ? p.plan.unit_seq[u + (int)num_clusters_x()] : 0;
    }
    valid = false;
  }
  __device__ __forceinline__ void init(const Params& p) {
    u = (int)cluster_id_x();
    g = 0;
    seg = 0;
    b = u < p.plan.header[1] ? p.plan.unit_seq[u] : 0;
    find(p);
  }
  __device__ __forceinline__ void next(const Params& p) {
    ++g;
    if (++k < nk) return;
    ++seg;
    ++b;
    if (enter_sequence(p)) return;
    u += (int)num_clusters_x();
    b = u < p.plan.header[1] ? p.plan.unit_seq[u] : 0;
    find(p);
  }
  __device__ __forceinline__ int j() const { return j0 + kT * k; }
  __device__ __forceinline__ int rows() const { return min(kT, j1 - j()); }
  __device__ __forceinline__ bool first() const { return k == 0; }
  __device__ __forceinline__ bool last() const { return k == nk - 1; }
  // cache rows attention row `row` sees: new token t of q_len sits at len - q_len + t and does
  // not see the new tokens after it
  __device__ __forceinline__ int visible(const Params& p, int row) const {
    return len - (p.q_len - 1 - (p.row_base + row) / p.heads_per_token);
  }
  // the query row of attention row `row` (576 values), or nullptr past the launch's rows
  __device__ __forceinline__ const __nv_bfloat16* q_row(const Params& p, int row) const {
    return row < p.n_heads ? p.q_abs + ((int64_t)b * p.q_row_stride + p.row_base + row) * kRow : nullptr;
  }
};

// Prefill: this cluster's work items (item u: sequence b, head, token block tb; items
// cluster_id, cluster_id + clusters, ...), each one segment over the cache rows its block's
// last token sees. Attention row r of an item is new token t = 128 tb + r of the head.
struct PrefillCursor {
  int u, b, head, tb;
  int slot, len, j0, j1;   // slot: the item; len: the sequence's kv_len
  int k, nk;
  uint32_t g, seg;
  bool valid;

  __device__ __forceinline__ void find(const Params& p) {
    if (u < p.n_items) {
      tb = u % p.n_blocks;
      head = (u / p.n_blocks) % p.heads_per_token;
      b = u / (p.n_blocks * p.heads_per_token);
      len = (int)min(max((int64_t)p.kv_lens[b], (int64_t)0), p.max_kv_len);
      slot = u;
      j0 = 0;
      j1 = max(0, min(len, len - p.q_tokens + 128 * (tb + 1)));
      // an item whose rows see nothing still takes one (empty) tile: its rows get latent 0 and
      // lse -inf from the same code as every other row
      nk = max(1, (j1 + kT - 1) / kT);
      k = 0;
      valid = true;
    } else {
      valid = false;
    }
  }
  __device__ __forceinline__ void init(const Params& p) {
    u = (int)cluster_id_x();
    g = 0;
    seg = 0;
    find(p);
  }
  __device__ __forceinline__ void next(const Params& p) {
    ++g;
    if (++k < nk) return;
    ++seg;
    u += (int)num_clusters_x();
    find(p);
  }
  __device__ __forceinline__ int j() const { return j0 + kT * k; }
  __device__ __forceinline__ int rows() const { return min(kT, j1 - j()); }
  __device__ __forceinline__ bool first() const { return k == 0; }
  __device__ __forceinline__ bool last() const { return k == nk - 1; }
  __device__ __forceinline__ int visible(const Params& p, int row) const {
    const int t = 128 * tb + row;
    return t < p.q_tokens ? len - p.q_tokens + t + 1 : 0;
  }
  __device__ __forceinline__ const __nv_bfloat16* q_row(const Params& p, int row) const {
    const int t = 128 * tb + row;
    return t < p.q_tokens ? p.q_abs + (((int64_t)b * p.q_tokens + t) * p.heads_per_token + head) * kRow : nullptr;
  }
};

__device__ __forceinline__ bool wait_teardown(uint32_t bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

// Query row h as an MMA operand: 16-byte chunks 0..31 (the CTA's 256 c^KV columns) go to
// TMEM columns kTmemQ + 4 chunk of the calling warp's lanes, chunks 32..35 (its 32 k^R
// columns) to row h of the shared-memory A operand of the k^R MMAs (64-byte swizzle).
__device__ __forceinline__ void q_chunks_out(const uint4 (&v)[12], uint8_t* smem, uint32_t tmem,
                                             uint32_t lanes, int h, int part) {
#pragma unroll
  for (int grp = 0; grp < 3; ++grp) {
    if (part == 2 && grp == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(smem + kOffQr + h * 64 + ((i ^ ((h >> 1) & 3)) << 4)) = v[8 + i];
    } else {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r[4 * i] = v[4 * grp + i].x; r[4 * i + 1] = v[4 * grp + i].y;
        r[4 * i + 2] = v[4 * grp + i].z; r[4 * i + 3] = v[4 * grp + i].w;
      }
      tmem_st16(lanes | (tmem + kTmemQ + 16 * (3 * part + grp)), r);
    }
  }
}

// One third (12 of the 36 16-byte chunks) of this CTA's 288 query columns of attention row h
// (query row qrow, or zeros when it is nullptr), to TMEM / shared memory as above.
__device__ __forceinline__ void load_q_part(const __nv_bfloat16* qrow, uint8_t* smem, uint32_t tmem,
                                            uint32_t lanes, int h, int part, uint32_t rank) {
  uint4 v[12];
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const int ci = part * 12 + i;  // 16-byte chunk 0..35 of this CTA's 288 columns
    const int col = ci < 32 ? 256 * (int)rank + 8 * ci : kDLatent + 32 * (int)rank + 8 * (ci - 32);
    v[i] = qrow != nullptr ? *reinterpret_cast<const uint4*>(qrow + col) : make_uint4(0, 0, 0, 0);
  }
  q_chunks_out(v, smem, tmem, lanes, h, part);
}

// The same third of the first segment's query columns, from the TMA copy in stages 1-2
// (row h of each box, 16-byte chunks under the boxes' 128- and 64-byte swizzles).
__device__ __forceinline__ void q_part_from_smem(uint8_t* smem, uint32_t tmem, uint32_t lanes,
                                                 int h, bool head_ok, int part) {
  const uint8_t* q = smem + kStageBytes;
  uint4 v[12];
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const int ci = part * 12 + i;
    const uint32_t off = ci < 32
        ? (uint32_t)(ci >> 3) * kQBoxC + (uint32_t)h * 128 + (uint32_t)(((ci & 7) ^ (h & 7)) << 4)
        : 4 * kQBoxC + (uint32_t)h * 64 + (uint32_t)((((ci - 32) & 3) ^ ((h >> 1) & 3)) << 4);
    v[i] = head_ok ? *reinterpret_cast<const uint4*>(q + off) : make_uint4(0, 0, 0, 0);
  }
  q_chunks_out(v, smem, tmem, lanes, h, part);
}

#include "e4m3_expand.cuh"   // the quantised cache's in-place expansion


// Rare paths of the softmax loop, kept out of line so that the loop's code stays small.
__device__ __noinline__ void rescale_o(uint32_t taddr, float alpha) {
#pragma unroll 1
  for (int cc = 0; cc < 8; ++cc) {
    uint32_t o[32];
    tmem_ld32_sync(taddr + kTmemO + 32 * cc, o);
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
    tmem_st32(taddr + kTmemO + 32 * cc, o);
  }
}

__device__ __noinline__ void zero_tail(uint8_t* stage, int r, int tid) {
  for (int i = tid; i < (kT - r) * 32; i += 128) {
    const int row = r + (i >> 5), box = (i >> 3) & 3, chunk = i & 7;
    *reinterpret_cast<uint4*>(stage + box * kBoxC + row * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
}

// kQ8: the cache is quantised (E4M3 codes expanded in shared memory); a separate
// instantiation, so that the bf16 kernel carries none of that code.
// kPrefill: the work is prefill items (PrefillCursor) instead of the split plan's segments,
// and each item's latent rows go straight to the output.
template <bool kQ8, bool kPrefill>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_split_tc(const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ CUtensorMap tmap_r,
                const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_qr,
                const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kOffBars;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* tile_valid = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);  // [kStages]
  volatile long long* tile_row_s = reinterpret_cast<volatile long long*>(smem + kOffMisc + 24);  // [kStages]
  constexpr bool q8 = kQ8;   // quantised cache
  using Cursor = std::conditional_t<kPrefill, PrefillCursor, TileCursor>;
  float2* ml = reinterpret_cast<float2*>(smem + kOffMl);                             // [2][2][128]
  volatile float* mh = reinterpret_cast<volatile float*>(smem + kOffMh);             // [128]
  volatile int* epi_seg = reinterpret_cast<volatile int*>(smem + kOffEpi);           // [128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(kBarKvFull + i), 1);
      mbar_init(bar(kBarKvEmpty + i), 1);
      tile_valid[i] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), 128);
      mbar_init(bar(kBarPFull + i), 128);
      mbar_init(bar(kBarPvDone + i), 1);
      mbar_init(bar(kBarPvDone + 2 + i), 1);
    }
    mbar_init(bar(kBarFinal2), 1);
    for (int i = 0; i < 16; ++i) mbar_init(bar(kBarXFull + i), 1);
    mbar_init(bar(kBarQReady), 128);
    mbar_init(bar(kBarQReady0), 384);
    mbar_init(bar(kBarQLanded), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(kBarMHand + i), 32);
    mbar_init(bar(kBarQFree), 1);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarOFree), 128);
    mbar_init(bar(kBarMlFull), 256);
    mbar_init(bar(kBarMlFull1), 256);
    for (int i = 0; i < kStages; ++i) mbar_init(bar(kBarKvConv + i), 128);
    mbar_init(bar(kBarConvSync), 128);
    for (int i = 0; i < 128; ++i) epi_seg[i] = 0;
    mbar_init(bar(kBarFinal), 1);
    *abort_flag = 0;
    // every softmax warp's block of both buffers expects its first tile of partial scores
    for (int i = 0; i < 16; ++i) mbar_arrive_expect_tx(bar(kBarXFull + i), kXBlockBytes);
    fence_mbarrier_init_cluster();
    prefetch_tmap(&tmap_c);
    prefetch_tmap(&tmap_r);
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_qr);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  cluster_sync();  // the peer's barriers are initialised before anyone signals them
  grid_dependency_wait();   // the plan, the query and the cache come from earlier kernels
  allow_dependent_launch();

  const WaitGuard guard{abort_flag, p.err, kErrTimeout, p.wait_limit};

  if (warp < 4) regs_dec<kRegsCtrl>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // first row of a tile in the cache, or -1 for a page-table entry out of range
      auto tile_row = [&](const Cursor& t) -> int64_t {
        const int j = t.j();
        if (p.page_table == nullptr) return (int64_t)t.b * p.seq_stride + j;
        const int32_t page = p.page_table[(int64_t)t.b * p.max_pages + j / kTileTokens];
        if (page < 0 || page >= p.num_pages) return -1;
        return (int64_t)page * kTileTokens + (j % kTileTokens);
      };
      Cursor c;
      c.init(p);
      // decode reads each cache tile once: its lines may leave L2 first, ahead of the split
      // partials the combine reads next (prefill items of other heads re-read the same rows)
      const uint64_t pol = kPrefill ? l2_policy_evict_normal() : l2_policy_evict_first();
      if (c.valid) {   // the first segment's query columns: one request, ahead of the tiles
        const uint32_t qdst = sbase + kStageBytes;
        mbar_arrive_expect_tx(bar(kBarQLanded), kQBytes);
        if constexpr (kPrefill) {   // 128 tokens of one head: (column, head, token) maps
          const int tok = c.b * p.q_tokens + 128 * c.tb;
          for (int i = 0; i < 4; ++i)
            tma_load_3d(qdst + i * kQBoxC, &tmap_q, 256 * (int)rank + 64 * i, c.head, tok, bar(kBarQLanded));
          tma_load_3d(qdst + 4 * kQBoxC, &tmap_qr, kDLatent + 32 * (int)rank, c.head, tok, bar(kBarQLanded));
        } else {
          const int qrow = c.b * p.q_row_stride + p.row_base;
          for (int i = 0; i < 4; ++i)
            tma_load_2d(qdst + i * kQBoxC, &tmap_q, 256 * (int)rank + 64 * i, qrow, bar(kBarQLanded));
          tma_load_2d(qdst + 4 * kQBoxC, &tmap_qr, kDLatent + 32 * (int)rank, qrow, bar(kBarQLanded));
        }
      }
      for (; c.valid; c.next(p)) {
        const uint32_t g = c.g, st = g % kStages;
        if (!wait_bounded(bar(kBarKvEmpty + st), ((g / kStages) & 1u) ^ 1u, guard)) break;
        // stages 1-2 hold the first segment's query until it is in TMEM
        if (g == 1 && !wait_bounded(bar(kBarQReady0), 0, guard)) break;
        const int64_t row = tile_row(c);
        const bool ok = row >= 0;
        if (!ok) atomicOr(p.err, kErrBadPage);
        tile_valid[st] = ok ? 1 : 0;
        tile_row_s[st] = row;
        const uint32_t dst = sbase + st * kStageBytes;
        if (ok && q8) {   // the codes, each box's into the upper half of its bf16 slot
          mbar_arrive_expect_tx(bar(kBarKvFull + st), kQ8StageBytes);
          for (int i = 0; i < 4; ++i)
            tma_load_2d_hint(dst + i * kBoxC + kBoxC / 2, &tmap_c, 256 * (int)rank + 64 * i, (int)row,
                             bar(kBarKvFull + st), pol);
          tma_load_2d_hint(dst + 4 * kBoxC + kBoxR / 2, &tmap_r, kDLatent + 32 * (int)rank, (int)row,
                           bar(kBarKvFull + st), pol);
        } else if (ok) {
          mbar_arrive_expect_tx(bar(kBarKvFull + st), kStageBytes);
          // the CTA's four 64-column c^KV boxes in one copy (3-D map: column, row, column group),
          // then its 32 k^R columns: two TMA instructions per tile keep the producer's warp
          // from crowding the softmax warps that share its SM sub-partition
          tma_load_3d_hint(dst, &tmap_c, 0, (int)row, 4 * (int)rank, bar(kBarKvFull + st), pol);
          tma_load_2d_hint(dst + 4 * kBoxC, &tmap_r, 32 * (int)rank, (int)row, bar(kBarKvFull + st), pol);
        } else {
          mbar_arrive(bar(kBarKvFull + st));
        }
      }
      // copies still in flight (only after an abort) land before the CTA leaves
      for (uint32_t i = 0; i < kStages && i < c.g; ++i) {
        const uint32_t gi = c.g - 1 - i;
        wait_teardown(bar(kBarKvFull + gi % kStages), (gi / kStages) & 1u, p.wait_limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK issuer
    // S(g) = Q . K(g)^T once the tile landed, the softmax has copied S(g-1) out of TMEM
    // and (first tile of a segment) the segment's query columns are in TMEM.
    if (lane == 0) {
      Cursor c;
      c.init(p);
      for (; c.valid; c.next(p)) {
        const uint32_t g = c.g, st = g % kStages;
        // the tile in bf16: landed, or (quantised cache) landed and expanded
        if (!wait_bounded(bar((q8 ? kBarKvConv : kBarKvFull) + st), (g / kStages) & 1u, guard)) break;
        // S is free once the softmax copied S(g-1) out (tile g-1's warpgroup)
        if (g > 0 && !wait_bounded(bar(kBarSEmpty + ((g - 1) & 1u)), ((g - 1) >> 1) & 1u, guard)) break;
        if (c.first() && !wait_bounded(c.seg == 0 ? bar(kBarQReady0) : bar(kBarQReady),
                                       c.seg == 0 ? 0u : (c.seg - 1) & 1u, guard))
          break;
        tc_fence_after();
        // One descriptor per operand region, stepped by adding the byte offset / 16 to its
        // start-address field (bits 0-13): shared addresses stay below 2^18, so the field never
        // carries into the next one. The issuing thread then spends one add per MMA instead of
        // rebuilding a 64-bit descriptor, which is what bounds how fast one thread can issue.
        const uint32_t a = sbase + st * kStageBytes;
        const uint64_t dc = smem_desc(a, 16, 1024, 2);             // the four c^KV boxes
        const uint64_t dr = smem_desc(a + 4 * kBoxC, 16, 512, 4);  // the k^R box
        const uint64_t dq = smem_desc(sbase + kOffQr, 16, 512, 4);  // the k^R query columns
#pragma unroll
        for (int ks = 0; ks < 16; ++ks)
          mma_ts(tmem + kTmemS, tmem + kTmemQ + 8 * ks, dc + (uint64_t)(((ks >> 2) * kBoxC + (ks & 3) * 32) >> 4),
                 kIdescQK, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ss(tmem + kTmemS, dq + (uint64_t)((ks * 32) >> 4), dr + (uint64_t)((ks * 32) >> 4), kIdescQK, 1u);
        mma_commit(bar(kBarSFull + (g & 1u)));
        if (c.last()) mma_commit(bar(kBarQFree));
      }
      mma_commit(bar(kBarFinal));
      wait_teardown(bar(kBarFinal), 0, p.wait_limit);
    }
  } else if (warp == 3) {
    // idle
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    // O += P(g) . V(g) once P(g) is in TMEM and (first tile of a segment) the previous
    // segment's O has been read out. Its completion frees the stage, P, and O.
    if (lane == 0) {
      Cursor c;
      c.init(p);
      for (; c.valid; c.next(p)) {
        const uint32_t g = c.g, st = g % kStages;
        if (!wait_bounded(bar(kBarPFull + (g & 1u)), (g >> 1) & 1u, guard)) break;
        if (c.first() && c.seg > 0 && !wait_bounded(bar(kBarOFree), (c.seg - 1) & 1u, guard)) break;
        tc_fence_after();
        const uint64_t dv = smem_desc(sbase + st * kStageBytes, kBoxC, 1024, 2);
        const uint32_t pcol = kTmemP + (kT / 2) * (g & 1u);
#pragma unroll
        for (int kk = 0; kk < kT / 16; ++kk)
          mma_ts(tmem + kTmemO, tmem + pcol + 8 * kk, dv + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                 (!c.first() || kk > 0) ? 1u : 0u);
        mma_commit(bar(kBarKvEmpty + st));
        mma_commit(bar(kBarPvDone + (g & 3u)));
        if (c.last()) mma_commit(bar(kBarOFull));
      }
      mma_commit(bar(kBarFinal2));
      wait_teardown(bar(kBarFinal2), 0, p.wait_limit);
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ softmax
    // Two warpgroups take alternate tiles (wg = g % 2); a thread owns one head (its TMEM lane)
    // and all 64 tokens of its warpgroup's tiles, so each warpgroup has two tile periods for a
    // tile's fetch, exchange, exponentials and P. The running max passes from one tile to the
    // next through shared memory and an mbarrier per head quarter (handoff k: tile k to k+1,
    // produced only after handoff k-1 was consumed, so its phase parity is unambiguous); each warpgroup
    // keeps its own share of the normaliser (relative to the max it last used), and the
    // epilogue merges the two.
    regs_inc<kRegsSoftmax>();
    const int quarter = warp & 3;                       // TMEM lanes this warp may touch
    const int wg = (warp >> 2) - 1;                     // the tiles of parity wg are ours
    const int h = 32 * quarter + lane;                  // head = TMEM lane
    const uint32_t lanes = (uint32_t)(32 * quarter) << 16;
    const int tid = threadIdx.x - 128 - 128 * wg;       // 0..127 within the warpgroup
    const uint32_t mhand = bar(kBarMHand + quarter);     // running-max handoff of these heads
    const uint32_t xin = sbase + kOffXin;
    const uint32_t peer_xin = map_to_rank(xin, peer);
    const int xbar0 = kBarXFull + 8 * wg + quarter;     // + 4 * buffer
    const uint32_t peer_xfull = map_to_rank(bar(xbar0), peer);   // + 32 bytes per buffer
    const uint32_t blk = (uint32_t)quarter * kXBlockBytes;
    const uint32_t rowoff = blk + (uint32_t)lane * 128;          // this head's 64 scores
    const uint32_t expoff = blk + 32 * 128 + (uint32_t)lane * 4; // ... and their scale
    auto xbuf = [&](uint32_t i) { return (uint32_t)(2 * wg + (int)i) * kXBufBytes; };

    // Block floating point for the exchange: with 2^(e-1) <= max|s| < 2^e each score becomes
    // k = round(s * 2^(14-e)) (|k| <= 2^14), within 2^-15 of the row's power-of-two ceiling; a
    // row holding a non-finite score is sent as all-NaN (kNonFinite). No int/float conversion
    // instructions (a quarter-rate pipe): fma(s, 2^(14-e), 2^23 + 2^15) rounds to the integer
    // 2^23 + 2^15 + k, whose low 16 bits are k + 2^15; the receiver rebuilds the float
    // 2^23 + (k + 2^15) from them with one byte permute and takes k * 2^(e-14) with one fma.
    constexpr int kNonFinite = 1000;
    constexpr float kMagic = 8421376.f;   // 2^23 + 2^15
    auto quantize = [&](const float (&v)[kT], uint32_t (&q)[kT / 2]) -> int {
      float am[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) am[i] = 0.f;
#pragma unroll
      for (int j = 0; j < kT; ++j)   // max.NaN: a NaN anywhere survives into amax
        asm("max.NaN.f32 %0, %0, %1;" : "+f"(am[j & 7]) : "f"(fabsf(v[j])));
#pragma unroll
      for (int i = 1; i < 8; ++i) asm("max.NaN.f32 %0, %0, %1;" : "+f"(am[0]) : "f"(am[i]));
      const float amax = am[0];
      const int eb = (int)((__float_as_uint(amax) >> 23) & 0xffu);
      const int e = max(eb - 126, -100);
      const float up = __uint_as_float((uint32_t)(141 - min(e, 128)) << 23);   // 2^(14 - e)
#pragma unroll
      for (int j = 0; j < kT / 2; ++j) {
        const float2 y = ffma2(make_float2(v[2 * j], v[2 * j + 1]), make_float2(up, up), make_float2(kMagic, kMagic));
        q[j] = __byte_perm(__float_as_uint(y.x), __float_as_uint(y.y), 0x5410);
      }
      return eb == 255 ? kNonFinite : e;
    };
    // Local tile u = g / 2 of this warpgroup lands in our buffer u % 2; our own block of tile u
    // is staged in buffer (u+1) % 2 and copied in one bulk transfer into the peer's buffer
    // u % 2. That is safe as soon as the peer's local tile u-1 has arrived here (awaited in
    // our previous local tile): the peer sent it only after our tile u-2 had reached it, so our
    // staging buffer (last used for tile u-2) has been read out and the peer is done with its
    // buffer u % 2 (it read our tile u-2 there; its own u-1 staged there has landed with us).
    auto send = [&](uint32_t u, const uint32_t (&q)[kT / 2], int e) {
      const uint32_t base = xin + xbuf((u + 1) & 1u);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(base + rowoff + (uint32_t)((c ^ (lane & 7)) * 16), q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
      asm volatile("st.shared.b32 [%0], %1;" :: "r"(base + expoff), "r"(e) : "memory");
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        bulk_copy_to_peer(peer_xin + xbuf(u & 1u) + blk, base + blk, kXBlockBytes,
                          peer_xfull + 32u * (u & 1u));
    };

    uint32_t total = 0;   // tiles of this cluster's work
    {
      Cursor t;
      t.init(p);
      if (t.valid) {   // two thirds of the first segment's query columns (the rest: transitions)
        if (wait_bounded(bar(kBarQLanded), 0, guard)) {
          q_part_from_smem(smem, tmem, lanes, h, h < p.n_heads, wg);
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(kBarQReady0));
      }
      for (; t.valid; t.next(p)) ++total;
    }
    Cursor c;
    c.init(p);
    float m_own = -INFINITY, l_own = 0.f;   // this warpgroup's max and normaliser share
    int my_seg = -1;                        // segment of the last tile this warpgroup took
    bool ok = true;
    uint32_t consumed = 0;                  // local tiles whose peer scores have been read
    for (; ok && c.valid; c.next(p)) {
      const uint32_t g = c.g;
      if ((int)(g & 1u) == wg) {
        const uint32_t st = g % kStages, u = g >> 1, xb = u & 1u;
        if (!wait_spin(bar(kBarKvFull + st), (g / kStages) & 1u, guard)) break;
        const int r = tile_valid[st] ? c.rows() : 0;   // valid tokens of the tile
        // ... of which this row sees those up to its own token's position
        const int rr = max(0, min(r, c.visible(p, h) - c.j()));
        // own partial S out of TMEM (S is free for the next QK once we have it)
        float sv[kT];
        {
          if (!wait_spin(bar(kBarSFull + wg), u & 1u, guard)) break;
          tc_fence_after();
          uint32_t a[32], b[32];
          tmem_ld32_sync(lanes | (tmem + kTmemS), a);
          tmem_ld32_sync(lanes | (tmem + kTmemS + 32), b);
          tc_fence_before();
          mbar_arrive(bar(kBarSEmpty + wg));
#pragma unroll
          for (int j = 0; j < 32; ++j) { sv[j] = __uint_as_float(a[j]); sv[32 + j] = __uint_as_float(b[j]); }
        }
        if (rr < kT) {   // the last tile of a sequence (or a skipped page): what is not there is 0 ...
#pragma unroll
          for (int j = 0; j < kT; ++j) sv[j] = j < rr ? sv[j] : 0.f;
        }
        {   // ... to the peer, then the peer's partial back: S = own + peer
          uint32_t qv[kT / 2];
          const int e = quantize(sv, qv);
          send(u, qv, e);
          const uint32_t xfull = bar(xbar0 + 4 * (int)xb);
          if (!wait_spin(xfull, (u >> 1) & 1u, guard)) break;
          if (lane == 0) mbar_arrive_expect_tx(xfull, kXBlockBytes);   // local tile u + 2
          const uint8_t* buf = smem + kOffXin + xbuf(xb);
          const int ep = *reinterpret_cast<const int*>(buf + expoff);
          const float down = ep != kNonFinite ? __uint_as_float((uint32_t)(113 + ep) << 23)
                                              : __int_as_float(0x7fc00000);
          const float bias = -kMagic * down;   // exact: both are powers-of-two multiples
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 v = *reinterpret_cast<const uint4*>(buf + rowoff + (uint32_t)((cc ^ (lane & 7)) * 16));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = __uint_as_float(__byte_perm(wv[i], 0x4B000000u, 0x7610));   // 2^23 + q
              const float hi = __uint_as_float(__byte_perm(wv[i], 0x4B000000u, 0x7632));
              const float2 t = ffma2(make_float2(lo, hi), make_float2(down, down), make_float2(bias, bias));
              const float2 r2 = fadd2(make_float2(sv[8 * cc + 2 * i], sv[8 * cc + 2 * i + 1]), t);
              sv[8 * cc + 2 * i] = r2.x;
              sv[8 * cc + 2 * i + 1] = r2.y;
            }
          }
          consumed = u + 1;
        }
        if (rr < kT) {
#pragma unroll
          for (int j = 0; j < kT; ++j) sv[j] = j < rr ? sv[j] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = sv[i];
#pragma unroll
        for (int j = 8; j < kT; ++j) mx[j & 7] = fmaxf(mx[j & 7], sv[j]);
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * p.scale_log2;

        // the running max after tile g-1, from the other warpgroup
        float m_prev = -INFINITY;
        if (g > 0) {
          if (!wait_spin(mhand, (g - 1) & 1u, guard)) break;
          m_prev = mh[h];
        }
        if (c.first()) m_prev = -INFINITY;          // a new segment starts from nothing
        if (my_seg != c.seg) { m_own = -INFINITY; l_own = 0.f; my_seg = c.seg; }
        float m_new = m_prev, alpha = 1.f;
        bool need = false;
        if (m_prev == -INFINITY) {
          m_new = mt;
        } else if (mt > m_prev + kRescaleThreshold) {   // rescale O only when the max grows a lot
          m_new = mt;
          need = true;
          alpha = ex2_approx(m_prev - mt);
        }
        mh[h] = m_new;
        if (g + 1 < total) mbar_arrive(mhand);
        if (m_own != m_new) {   // our share of the normaliser to the new max
          l_own = m_own == -INFINITY ? 0.f : l_own * ex2_approx(m_own - m_new);
          m_own = m_new;
        }
        // P = 2^(s * scale * log2(e) - m)
        // (with no live token yet every score is -inf and 2^-inf = 0, so no select is needed)
        const float neg_m = m_new != -INFINITY ? -m_new : 0.f;
        float2 sm[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sm[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kT / 2; ++j) {
          const float2 x = ffma2(make_float2(sv[2 * j], sv[2 * j + 1]), make_float2(p.scale_log2, p.scale_log2),
                                 make_float2(neg_m, neg_m));
          sv[2 * j] = ex2_approx(x.x);
          sv[2 * j + 1] = ex2_approx(x.y);
          sm[j & 3] = fadd2(sm[j & 3], make_float2(sv[2 * j], sv[2 * j + 1]));
        }
        l_own += ((sm[0].x + sm[0].y) + (sm[1].x + sm[1].y)) + ((sm[2].x + sm[2].y) + (sm[3].x + sm[3].y));
        const bool warp_need = __any_sync(0xffffffffu, need);

        // P(g) goes where P(g-2) was: PV(g-2) must be done (it nearly always is by now). O may be
        // rescaled only once PV(g-1) is done as well; without a rescale, PV(g-1) may still run.
        // PV(g) signals barrier g % 4: PV(g-4) is done (tile g's stage was refilled after it) and
        // PV(g+3) cannot be (it needs P(g)), so each of these waits is at most one phase behind
        // its barrier, which a phase parity can tell apart.
        if (g > 1 && !wait_spin(bar(kBarPvDone + ((g - 2) & 3u)), ((g - 2) >> 2) & 1u, guard)) break;
        if (warp_need && g > 0 && !wait_spin(bar(kBarPvDone + ((g - 1) & 3u)), ((g - 1) >> 2) & 1u, guard)) break;
        tc_fence_after();
        if (warp_need) rescale_o(lanes | tmem, alpha);   // O (all 256 columns of this head) to the new max
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {   // P as bf16 pairs, 32 columns
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(sv[32 * hf + 2 * j], sv[32 * hf + 2 * j + 1]);
            pk[j] = *reinterpret_cast<uint32_t*>(&b2);
          }
          tmem_st16(lanes | (tmem + kTmemP + (kT / 2) * wg + 16 * hf), pk);
        }
        tmem_wait_st();
        if (r < kT) zero_tail(smem + st * kStageBytes, r, tid);   // rows past the end must not reach P.V
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + wg));
      }
      if (c.last()) {   // segment done: this warpgroup's (max, share) for the epilogue
        const bool mine = my_seg == c.seg;
        // ml[seg % 2] was last read by the epilogue of segment seg - 2: wait for that read (a
        // per-head counter, since the softmax may be more than one segment ahead of it)
        if (c.seg >= 2) {
          const long long t0 = clock64();
          while (epi_seg[h] < (int)c.seg - 1) {
            if (*abort_flag) { ok = false; break; }
            if (clock64() - t0 > p.wait_limit) {
              atomicOr(p.err, kErrTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
          }
          if (!ok) break;
        }
        ml[((c.seg & 1u) * 2 + wg) * 128 + h] = make_float2(mine ? m_own : -INFINITY, mine ? l_own : 0.f);
        mbar_arrive(bar((c.seg & 1u) ? kBarMlFull1 : kBarMlFull));
      }
    }
    // after an abort: blocks the peer may still have in flight to us (it sends local tile u
    // once our u-1 arrived) land before we leave
    {
      uint32_t nloc = 0;   // local tiles of this warpgroup
      for (uint32_t t = (uint32_t)wg; t < total; t += 2) ++nloc;
      for (uint32_t t = consumed; t < consumed + 2 && t < nloc; ++t)
        wait_teardown(bar(xbar0 + 4 * (int)(t & 1u)), (t >> 1) & 1u, p.wait_limit >> 10);
    }
  } else {
    // ------------------------------------------------------------ segment transitions
    regs_dec<kRegsTrans>();
    const int quarter = warp & 3;
    const int h = 32 * quarter + lane;
    const uint32_t lanes = (uint32_t)(32 * quarter) << 16;
    const bool head_ok = h < p.n_heads;
    Cursor c;
    c.init(p);
    int prev_slot = -1;
    auto epilogue = [&](uint32_t seg, int slot) -> bool {
      if (!wait_bounded(bar(kBarOFull), seg & 1u, guard)) return false;
      if (!wait_bounded(bar((seg & 1u) ? kBarMlFull1 : kBarMlFull), (seg >> 1) & 1u, guard)) return false;
      tc_fence_after();
      const float2 m0 = ml[((seg & 1u) * 2 + 0) * 128 + h];
      const float2 m1 = ml[((seg & 1u) * 2 + 1) * 128 + h];
      __threadfence_block();
      epi_seg[h] = (int)seg + 1;   // both warpgroups may now overwrite ml[seg % 2] for this head
      // O is relative to the last max used (the larger: the max only grows); each warpgroup's
      // share of the normaliser is relative to the max it used last
      const float mlast = fmaxf(m0.x, m1.x);
      const float l0 = m0.y > 0.f ? m0.y * exp2f(m0.x - mlast) : 0.f;
      const float l1 = m1.y > 0.f ? m1.y * exp2f(m1.x - mlast) : 0.f;
      const float2 mls = make_float2(mlast, l0 + l1);
      const float inv = mls.y > 0.f ? 1.f / mls.y : 0.f;
      const float lse_e = mls.y > 0.f ? (mls.x + log2f(mls.y)) * 0.69314718055994531f : -INFINITY;
      if constexpr (kPrefill) {
        // the item's row h is new token t of the head: its normalised latent (this CTA's 256
        // columns) and lse go straight to the output
        const int tb = slot % p.n_blocks, head = (slot / p.n_blocks) % p.heads_per_token;
        const int b = slot / (p.n_blocks * p.heads_per_token);
        const int t = 128 * tb + h;
        const bool row_ok = t < p.q_tokens;
        const int64_t orow = ((int64_t)b * p.q_tokens + (row_ok ? t : 0)) * p.heads_per_token + head;
        __nv_bfloat16* dst = p.out_latent + orow * kDLatent + 256 * rank;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[32];
          tmem_ld32_sync(lanes | (tmem + kTmemO + 32 * cc), o);
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[8 * q + 2 * i]) * inv,
                                                          __uint_as_float(o[8 * q + 2 * i + 1]) * inv);
                w[i] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(dst + 32 * cc + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        if (row_ok && rank == 0 && p.out_lse != nullptr) p.out_lse[orow] = lse_e;
        tc_fence_before();
        mbar_arrive(bar(kBarOFree));
        return true;
      }
      // partial O as [slot][column quad][head][4 floats]: the 32 heads of a warp write 512
      // contiguous bytes per store, marked to stay in L2 for the combine
      const uint64_t keep = l2_policy_evict_last();
      const int64_t quad_stride = (int64_t)p.n_heads * 4;
      float* dst = p.part_o + ((int64_t)slot * (kDLatent / 4) + 64 * rank) * quad_stride +
                   (head_ok ? h : 0) * 4;
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t o[32];
        tmem_ld32_sync(lanes | (tmem + kTmemO + 32 * cc), o);
        if (head_ok) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_global_v4_hint(dst + (8 * cc + q) * quad_stride,
                              make_float4(__uint_as_float(o[4 * q]) * inv, __uint_as_float(o[4 * q + 1]) * inv,
                                          __uint_as_float(o[4 * q + 2]) * inv, __uint_as_float(o[4 * q + 3]) * inv),
                              keep);
        }
      }
      if (head_ok && rank == 0) p.part_lse[(int64_t)slot * p.n_heads + h] = lse_e;
      tc_fence_before();
      mbar_arrive(bar(kBarOFree));
      return true;
    };
    // Quantised cache: expand tile g's codes in place (see read_codes), then let its QK go.
    uint32_t n_expanded = 0;
    auto expand_tile = [&](uint32_t g) -> bool {
      const uint32_t st = g % kStages;
      if (!wait_bounded(bar(kBarKvFull + st), (g / kStages) & 1u, guard)) return false;
      const int t = (int)threadIdx.x - 384;   // 0..127 within this warpgroup
      const int64_t row0 = tile_row_s[st];
      const int64_t row = row0 + (t >> 1);
      const int e = (row0 >= 0 && row < p.kv_rows) ? min(max((int)p.kv_exp[row], -126), 127) : 0;
      uint8_t* stage = smem + st * kStageBytes;
      TileCodes v;
      read_codes(stage, t, v);
      mbar_arrive(bar(kBarConvSync));
      if (!wait_bounded(bar(kBarConvSync), n_expanded & 1u, guard)) return false;
      ++n_expanded;
      write_bf16(stage, t, v, e);
      fence_proxy_async_smem();   // read by the MMAs (async proxy)
      mbar_arrive(bar(kBarKvConv + st));
      return true;
    };
    bool ok = true;
    while (ok && c.valid) {
      const uint32_t seg = c.seg;
      // this segment's query columns -> TMEM, once the previous segment's last QK is done
      if (seg > 0 && !wait_bounded(bar(kBarQFree), (seg - 1) & 1u, guard)) break;
      tc_fence_after();
      {
        if (seg == 0) {
          // the first segment's query: the softmax warps load the other two thirds, so the
          // three batches of loads overlap instead of queueing behind the first cache tiles
          if (wait_bounded(bar(kBarQLanded), 0, guard)) {
            q_part_from_smem(smem, tmem, lanes, h, head_ok, 2);
            tmem_wait_st();
            fence_proxy_async_smem();
          }
          tc_fence_before();
          mbar_arrive(bar(kBarQReady0));
        } else {
          const __nv_bfloat16* qrow = c.q_row(p, h);
#pragma unroll 1
          for (int part = 0; part < 3; ++part) load_q_part(qrow, smem, tmem, lanes, h, part, rank);
          tmem_wait_st();
          fence_proxy_async_smem();   // the k^R query columns are read by the MMA (async proxy)
          tc_fence_before();
          mbar_arrive(bar(kBarQReady));
        }
      }
      // the previous segment's output, while this one runs (with a quantised cache, after
      // this segment's first tile is expanded, so that its QK does not wait for the epilogue)
      if (seg > 0 && !q8) ok = epilogue(seg - 1, prev_slot);
      const int seg_slot = c.slot;
      // walk to the next segment (expanding each quantised tile on the way), and pull its
      // query rows into L2 while this one runs
      bool first_tile = true;
      while (ok && c.valid && c.seg == seg) {
        if (q8) {
          if (!expand_tile(c.g)) { ok = false; break; }
          if (first_tile && seg > 0) ok = epilogue(seg - 1, prev_slot);
        }
        first_tile = false;
        c.next(p);
      }
      prev_slot = seg_slot;
      if (!ok) break;
      const __nv_bfloat16* qrow = c.valid ? c.q_row(p, h) : nullptr;
      if (qrow != nullptr) {
        asm volatile("prefetch.global.L2 [%0];" :: "l"(qrow + 256 * (int)rank) : "memory");
        asm volatile("prefetch.global.L2 [%0];" :: "l"(qrow + 256 * (int)rank + 64) : "memory");
        asm volatile("prefetch.global.L2 [%0];" :: "l"(qrow + 256 * (int)rank + 128) : "memory");
        asm volatile("prefetch.global.L2 [%0];" :: "l"(qrow + 256 * (int)rank + 192) : "memory");
        asm volatile("prefetch.global.L2 [%0];" :: "l"(qrow + kDLatent + 32 * (int)rank) : "memory");
      }
      if (!c.valid && ok) ok = epilogue(seg, prev_slot);
    }
  }

  // teardown: nobody touches the peer's shared memory after this point
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// c^KV as a 3-D tensor (64 columns, rows, 8 column groups of 64): one box {64, 64, 4} is four
// consecutive 64x64 boxes in shared memory, each row 128 bytes under the 128-byte swizzle.
bool encode_latent_groups(CUtensorMap* m, const void* base, uint64_t rows, int64_t row_stride) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {64, rows, kDLatent / 64};
  const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, 128};
  const cuuint32_t box[3] = {64, (cuuint32_t)kT, 4};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, int64_t row_stride,
                 uint32_t box_cols, CUtensorMapSwizzle swz, uint32_t box_rows = kT) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The quantised cache's codes as a 2-D byte tensor [rows, 576] with {box_cols, 64} boxes, no
// swizzle: a box lands as 64 dense rows of box_cols bytes.
bool encode_codes(CUtensorMap* m, const void* base, uint64_t rows, int64_t row_stride_bytes,
                  uint32_t box_cols) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, (cuuint32_t)kT};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q_abs [B, T, n_h, 576] as a 3-D tensor (columns, heads, tokens): a {box_cols, 1, 128} box is
// 128 consecutive tokens of one head and lands as 128 rows of box_cols columns.
bool encode_tokens(CUtensorMap* m, const void* base, uint64_t heads, uint64_t tokens, uint32_t box_cols,
                   CUtensorMapSwizzle swz) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kRow, heads, tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)kRow * 2, (cuuint64_t)heads * kRow * 2};
  const cuuint32_t box[3] = {box_cols, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t set_smem_attributes() {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(decode_split_tc<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemAlloc);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(decode_split_tc<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kSmemAlloc);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(decode_split_tc<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kSmemAlloc);
  });
  return attr_err;
}

}  // namespace

cudaError_t launch_prefill(const mla_decode_s& h, int batch, const __nv_bfloat16* q_abs,
                           const CacheView& cv, __nv_bfloat16* out_latent, float* lse, cudaStream_t s) {
  const cudaError_t attr = set_smem_attributes();
  if (attr != cudaSuccess) return attr;
  if (cv.kv_exp != nullptr) return cudaErrorInvalidValue;
  const int64_t rows = cv.page_table != nullptr ? (int64_t)cv.num_pages * cv.page_size
                                                : (int64_t)batch * cv.seq_stride;
  if (rows <= 0 || rows >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  const int T = h.q_len, n_h = h.cfg.n_heads;
  CUtensorMap tc, tr, tq, tqr;
  if (!encode_latent_groups(&tc, cv.c_kv, (uint64_t)rows, cv.row_stride) ||
      !encode_rows(&tr, cv.k_r, kDRope, (uint64_t)rows, cv.row_stride, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_tokens(&tq, q_abs, (uint64_t)n_h, (uint64_t)batch * T, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tokens(&tqr, q_abs, (uint64_t)n_h, (uint64_t)batch * T, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  Params p{};
  p.q_abs = q_abs;
  p.batch = batch;
  p.n_heads = 128;           // attention rows per item: 128 tokens of one head
  p.q_len = T;
  p.heads_per_token = n_h;
  p.row_base = 0;
  p.q_row_stride = T * n_h;
  p.seq_stride = cv.seq_stride;
  p.page_table = cv.page_table;
  p.max_pages = cv.max_pages;
  p.num_pages = cv.num_pages;
  p.scale_log2 = h.scale * 1.4426950408889634f;
  p.part_o = h.ws.part_o;
  p.part_lse = h.ws.part_lse;
  p.err = h.ws.err;
  p.wait_limit = 2000000000LL;  // SM cycles, about a second
  p.kv_exp = nullptr;
  p.kv_rows = rows;
  p.q_tokens = T;
  p.n_blocks = (T + 127) / 128;
  p.n_items = batch * n_h * p.n_blocks;
  p.kv_lens = cv.kv_lens;
  p.max_kv_len = h.cfg.max_kv_len;
  p.out_latent = out_latent;
  p.out_lse = lse;
  const int pairs = std::max(1, std::min(p.n_items, h.num_sms / 2));
  return launch_pdl(decode_split_tc<false, true>, dim3(2 * pairs), dim3(kThreads), kSmemAlloc, s, tc, tr, tq,
                    tqr, p);
}

cudaError_t launch_decode_split(const mla_decode_s& h, int batch, const __nv_bfloat16* q_abs,
                                const CacheView& cv, int row_base, cudaStream_t s) {
  const cudaError_t attr_err = set_smem_attributes();
  if (attr_err != cudaSuccess) return attr_err;

  const int64_t rows = cv.page_table != nullptr ? (int64_t)cv.num_pages * cv.page_size
                                                : (int64_t)batch * cv.seq_stride;
  if (rows <= 0 || rows >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  CUtensorMap tc, tr, tq, tqr;
  const uint64_t qrows = (uint64_t)batch * h.n_rows;   // q_abs as [B * rows, 576]
  const bool cache_ok =
      cv.kv_exp != nullptr
          ? encode_codes(&tc, cv.c_kv, (uint64_t)rows, cv.row_stride, 64) &&
                encode_codes(&tr, cv.c_kv, (uint64_t)rows, cv.row_stride, 32)
          : encode_latent_groups(&tc, cv.c_kv, (uint64_t)rows, cv.row_stride) &&
                encode_rows(&tr, cv.k_r, kDRope, (uint64_t)rows, cv.row_stride, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  if (!cache_ok ||
      !encode_rows(&tq, q_abs, kRow, qrows, kRow, 64, CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !encode_rows(&tqr, q_abs, kRow, qrows, kRow, 32, CU_TENSOR_MAP_SWIZZLE_64B, 128))
    return cudaErrorInvalidValue;

  Params p{};
  p.q_abs = q_abs;
  p.plan = h.ws.plan;
  p.batch = batch;
  p.n_heads = std::min(h.group_rows, h.n_rows - row_base);
  p.row_base = row_base;
  p.q_row_stride = h.n_rows;
  p.q_len = h.q_len;
  p.heads_per_token = h.cfg.n_heads;
  p.seq_stride = cv.seq_stride;
  p.page_table = cv.page_table;
  p.max_pages = cv.max_pages;
  p.num_pages = cv.num_pages;
  p.scale_log2 = h.scale * 1.4426950408889634f;
  p.part_o = h.ws.part_o;
  p.part_lse = h.ws.part_lse;
  p.err = h.ws.err;
  p.wait_limit = 2000000000LL;  // SM cycles, about a second
  p.kv_exp = cv.kv_exp;
  p.kv_rows = rows;

  const int pairs = std::max(1, std::min(h.units, h.num_sms / 2));
  // the 2-CTA cluster shape is compiled into the kernel
  return cv.kv_exp != nullptr
             ? launch_pdl(decode_split_tc<true, false>, dim3(2 * pairs), dim3(kThreads), kSmemAlloc, s, tc, tr, tq, tqr, p)
             : launch_pdl(decode_split_tc<false, false>, dim3(2 * pairs), dim3(kThreads), kSmemAlloc, s, tc, tr, tq, tqr, p);
}

}  // namespace mla
