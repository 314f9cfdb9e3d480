// Multi-token paged attention with a causal mask on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory), sm_100a.
//
// Same operation as prefill_tc.cu ("vLLM 0.5 深度拆解" §2.3 chunked prefill,
// "vLLM 推理引擎源码级拆解" §4.2 prefix-cache continuation, the §2.3 block-table
// walk): row r of a chunk of q_i query tokens sits at position seq_lens[i] - q_i
// + r and attends over tokens 0..pos of its sequence.
//
// How:
//  * The work is items of 256 query rows — (token, query head of the group)
//    pairs of one (sequence, KV head) — each two tiles of 128, each tile the M
//    of one tcgen05.mma. The kernel is persistent: one CTA per SM takes items
//    from a work counter as it becomes free, the items of a few (sequence, KV
//    head) pairs at a time, longest causal ranges first within them, so their
//    K/V stays in L2 and the shortest items come last. Within a CTA every role
//    walks the same sequence of items and 64-token chunks, so a chunk's place
//    in it names its K/V stage, S buffer and barrier phases in every role,
//    and the next item's Q and K/V stream in while the current one finishes.
//  * Eleven warps: eight softmax warps (warp w serves tile w / 4 and owns
//    tensor-memory lanes 32 (w % 4) .. +31, one row per thread), a TMA
//    producer warp and one MMA warp per tile (each runs its tile's issue loop
//    on warp-uniform operands; one elected thread issues every MMA and commit).
//    With two issuing warps on different sub-partitions, one warp's barrier
//    waits overlap the other's MMAs, so the tensor pipe rarely runs dry.
//  * The producer takes items from the counter, publishes their records to the
//    other roles through a small ring in shared memory, starts each item's Q
//    on its way into L2, and streams the causal range of each item in 64-token
//    chunks through a four-stage ring shared by both tiles. Each (block, KV
//    head) tile is copied as one TMA box per 64-element piece of head_dim, so
//    in shared memory a chunk's K (and V) is, per piece, 64 token rows of 128
//    bytes in the 128B swizzle: K is a K-major operand and V an MN-major
//    operand of the tensor core as it lands. A tile's Q (when g divides 128,
//    whole tokens) is one TMA box per piece of head_dim in the same layout,
//    loaded by one softmax thread as soon as the tile's last S of the previous
//    item has completed; otherwise the softmax threads copy their rows.
//  * An E4M3 cache: the producer copies a chunk's codes by TMA into a staging
//    ring (one chunk ahead); the producer widens K and a twelfth warp
//    widens V, exactly, to f16 in the chunk's stage, in the layout the 16-bit
//    path gets from TMA (the widening is bound by the issue rate of the warps
//    doing it, so it is split over two sub-partitions); the MMAs are f16 (Q
//    rounded to f16 by the softmax threads as they stage it), k_scale is folded
//    into the score scale and v_scale into the output.
//  * Each tile has two S buffers in tensor memory (chunk j uses buffer j % 2):
//    S = Q K^T of the next chunk (M 128, N 64, K 16 per instruction) is
//    computed into one while the softmax threads work on the other, so a
//    softmax thread finds its next S ready instead of waiting for it. The
//    threads read S with tcgen05.ld, apply the causal mask (only in chunks that
//    reach past a row's position) and the scale, keep a running maximum that
//    is only raised (and O rescaled in tensor memory) when a chunk's maximum
//    exceeds it by more than 2^8, so rescaling is rare and P = 2^(s - m) stays
//    below 256, and sum the rounded P into their row sums.
//  * P goes back over the first 32 columns of its own S buffer as 16-bit pairs,
//    and O += P V (A from tensor memory, M 128, N head_dim) accumulates in the
//    tile's O columns. A tile's MMA warp issues, per chunk j, the PV of chunk
//    j and then S of chunk j + 2 (of the next item past this one's end) into
//    the buffer that PV reads: the MMAs of a thread run in issue order, so
//    S(j + 2) overwrites P(j) only after the PV that read it. A K/V stage is
//    free once both tiles' warps have committed their PV of it. Once an
//    item's last PV has completed each thread reads its row of O, divides by
//    its row sum and stores it: this epilogue runs after the next item's first
//    chunk has been through the softmax and before that chunk's P is
//    published, so the wait for the last PV overlaps useful work and the next
//    item's first PV, which overwrites O, cannot start before O has been read.
//  * The commit after S(j + 2) (past the last chunk, a commit alone) also
//    tells a tile's softmax that PV(j) has completed: it is what O's rescale
//    waits for. P has a barrier per S buffer, so a softmax that runs a chunk
//    ahead never completes a phase twice.
//  * Slots past the causal range are masked in S and zeroed in V before the
//    last PV, so stale or poisoned memory never reaches the output.
//  * Every wait is bounded; on expiry the CTA records it, stops, waits (bounded)
//    for its own copies and MMAs in flight, and frees its tensor memory.
#include <algorithm>
#include <atomic>
#include <climits>
#include <type_traits>

#include "common.cuh"
#include "prefill.cuh"
#include "tc_common.cuh"

namespace pkv {

__device__ int g_pf5_status = 0;  // bit 0: a wait expired; bit 1: a block id outside the pool
// Work counters of the tcgen05 prefill: per slot the next item to hand out and
// the CTAs that have finished; the last CTA of a launch puts both back to 0.
__device__ int g_pf5_sched[64][2];  // 64 = kSchedSlots

namespace pf {
namespace {

using namespace tcx;

constexpr int kChunk = 64;      // K/V tokens per stage = N of S
constexpr int kRows = 128;      // query rows per tile = M of every MMA
constexpr int kTiles = 2;       // tiles per CTA, sharing each K/V chunk
constexpr int kCtaRows = kTiles * kRows;
constexpr int kSoftWarps = 4 * kTiles;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;  // MMA warps kMmaWarp + t, one per tile
constexpr int kThreads = (kSoftWarps + 1 + kTiles) * 32;
// E4M3 caches: a twelfth warp widens each chunk's V while the producer widens
// its K (on the fourth sub-partition, so it costs no registers: three warps
// per sub-partition either way).
constexpr int kWidenWarp = kSoftWarps + 1 + kTiles;
constexpr int kThreads8 = kThreads + 32;
constexpr int kNS = 4;          // K/V stages
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of 64 values as a tree of three-input maxima (depth 4, 32 ops)
// instead of a chain of 63 dependent two-input ones.
__device__ __forceinline__ float max64(const float (&s)[64]) {
  float t[22], u[8];
#pragma unroll
  for (int i = 0; i < 21; ++i) t[i] = max3f(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
  t[21] = s[63];
#pragma unroll
  for (int i = 0; i < 7; ++i) u[i] = max3f(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  u[7] = t[21];
  return max3f(max3f(u[0], u[1], u[2]), max3f(u[3], u[4], u[5]), fmaxf(u[6], u[7]));
}

// One unit of work: the 256 query rows row0 .. row0 + 255 of (sequence, KV
// head) and the 64-token chunks of its causal range; a record with no chunks
// tells the other roles that the work is gone.
struct Item {
  int seq, h, q0, rows, row0, base_pos, kv_end, nchunks;
};
constexpr int kRing = 8;        // item records in flight from the producer to the other roles
constexpr int kPairGroup = 8;   // (sequence, KV head) pairs whose items are handed out together
constexpr int kSchedSlots = 64; // work counters, one per launch in flight

// E4M3 caches: 4 stages of widened K/V and 2 stages of codes (copied by TMA one
// chunk ahead of their widening; measured faster than 3 + 4), in the same
// shared memory.

template <int D, bool F8>
struct Cfg5 {
  static constexpr int kPlanes = D / 64;          // 128-byte pieces of head_dim
  static constexpr int kPlaneKV = kChunk * 128;   // one piece of a K (or V) chunk
  static constexpr int kKV = kPlanes * kPlaneKV;
  static constexpr int kStage = 2 * kKV;          // K pieces, then V pieces
  static constexpr int kPlaneQ = kRows * 128;
  static constexpr int kQ = kPlanes * kPlaneQ;    // Q of one tile
  // Tensor-memory columns: two S buffers of 64 columns per tile (chunk c uses
  // buffer c % 2, at 128 t + 64 (c % 2); P of the chunk is written, as 16-bit
  // pairs, over the first 32 columns of its buffer), and O of tile t at
  // 256 + t D.
  static constexpr uint32_t kColO = 256;
  static_assert(kColO + kTiles * D <= kTmemCols, "tensor memory per CTA");
  // full, empty, s_full [tile][buffer], p_full [tile][buffer], q_full [tile], o_done [tile],
  // drain; then item_full and item_empty [kRing] and the ring of item records
  static constexpr int kNSx = kNS;            // stages of 16-bit K/V
  static constexpr int kNS8x = F8 ? 2 : 0;    // stages of E4M3 codes
  static constexpr int kBars = 2 * kNSx + 6 * kTiles + 1;
  // F8: per stage the E4M3 codes of a chunk's K, then of its V, as they land
  // (rows of min(D, 128) bytes in the 128B (64B when D = 64) swizzle).
  static constexpr int kRowB8 = D < 128 ? D : 128;
  static_assert(kRowB8 == 64 || kRowB8 == 128, "E4M3 rows are one 64- or 128-byte box");
  static constexpr int kKV8 = kChunk * D;
  static constexpr int kStage8 = F8 ? 2 * kKV8 : 0;
  static constexpr int kSmem = 1024 + kNSx * kStage + kNS8x * kStage8 + kTiles * kQ + kBars * 8 +
                               2 * kNS8x * 8 + 16 + kRing * (16 + (int)sizeof(Item));
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA exceeds 227 KB");
};

__device__ __forceinline__ bool wait5(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_or_abort(bar, parity, abort, &g_pf5_status);
}

// Four E4M3 codes (one 32-bit word) widened exactly to two f16 pairs; the
// halves of the word are taken as 16-bit registers, so no shift is needed.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n"
      " cvt.rn.f16x2.e4m3x2 %1, b;\n}" : "=r"(lo), "=r"(hi) : "r"(w));
}

// Shared-memory matrix descriptor: 128B swizzle, 8-row groups 1024 bytes apart,
// `lbo` between 64-element pieces (MN-major operands).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with an fp32 accumulator: A and B
// bf16 (1) or f16 (0), A K-major, B K-major (0) or MN-major (1), shape M x N.
template <typename T>
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((std::is_same<T, __nv_bfloat16>::value ? 1u : 0u) << 7) |
         ((std::is_same<T, __nv_bfloat16>::value ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (tensor memory) [+]= A (shared memory) x B (shared memory).
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}

// D (tensor memory) [+]= A (tensor memory: row i in lane i, K packed two
// elements per column) x B (shared memory).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// True in exactly one thread of the (converged) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

#define PKV_TMEM_REGS32(r)                                                                   \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),     \
      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),          \
      "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),          \
      "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define PKV_TMEM_LD32 \
  "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
  "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(PKV_TMEM_LD32 : PKV_TMEM_REGS32(r) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive fp32 columns: two loads in flight, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t a[32], b[32];
  asm volatile(PKV_TMEM_LD32 : PKV_TMEM_REGS32(a) : "r"(taddr));
  asm volatile(PKV_TMEM_LD32 : PKV_TMEM_REGS32(b) : "r"(taddr + 32));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __uint_as_float(a[i]);
    v[32 + i] = __uint_as_float(b[i]);
  }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  uint32_t u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(v[i]);
  tmem_st32(taddr, u);
}

// Byte offset of 16-byte chunk j of row r in a 128B-swizzled region of 128-byte rows.
__device__ __forceinline__ uint32_t sw(int r, int j) {
  return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

// Item i of a launch: the (sequence, KV head) pairs in groups of kPairGroup,
// and within a group tile pair xr (counted from the end of the chunk, so the
// longest causal ranges come first) of each pair in turn. CTAs take items in
// this order as they become free, so the K/V of a few pairs is in use at a
// time (it stays in L2) and the shortest items come last.
__device__ __forceinline__ bool load_item(const PrefillParams& p, int num_seqs, int tiles, int i,
                                          Item& it) {
  const int Hkv = p.num_kv_heads, g = p.num_heads / Hkv;
  const int64_t per_group = (int64_t)kPairGroup * tiles;
  const int grp = (int)(i / per_group);
  const int pg = min(kPairGroup, num_seqs * Hkv - grp * kPairGroup);
  const int within = (int)(i - grp * per_group), xr = within / pg;
  const int pair = grp * kPairGroup + within - xr * pg;
  it.seq = pair / Hkv;
  it.h = pair - it.seq * Hkv;
  const int q1 = min(max(__ldg(p.query_start + it.seq + 1), 0), p.num_q_tokens);
  it.q0 = max(min(max(__ldg(p.query_start + it.seq), 0), q1), q1 - p.max_q_len);
  const int qn = q1 - it.q0;
  it.rows = qn * g;
  const int L = min(__ldg(p.seq_lens + it.seq), p.max_blocks_per_seq * p.block_size);
  it.row0 = (tiles - 1 - xr) * kCtaRows;
  if (qn <= 0 || it.row0 >= it.rows || L <= 0) return false;
  it.base_pos = L - qn;
  const int last_row = min(it.rows, it.row0 + kCtaRows) - 1;
  it.kv_end = min(L, it.base_pos + last_row / g + 1);
  if (it.kv_end <= 0) return false;
  it.nchunks = (it.kv_end + kChunk - 1) / kChunk;
  return true;
}

// The items of this CTA, as the producer publishes them in a ring of kRing
// records, and their chunks, in order. Every role walks the same sequence, so
// the position of a chunk in it (its index j) names the same K/V stage
// (j % kNS), S buffer (j % 2) and barrier phases in every role. All lanes of a
// warp call the methods; a record with no chunks ends the sequence.
struct Walk {
  const Item* ring;
  uint64_t* full;
  volatile int* abort;
  int ii, c, nchunks;  // item number, chunk within it, its chunks
  bool ok;             // a current chunk exists
  __device__ __forceinline__ const Item& it() const { return ring[ii % kRing]; }
  __device__ __forceinline__ void next_item() {
    ++ii;
    const int slot = ii % kRing;
    const bool w = __all_sync(0xffffffffu, wait5(full + slot, (uint32_t)(ii / kRing) & 1u, abort));
    nchunks = w ? ring[slot].nchunks : 0;
    ok = nchunks > 0;
    c = 0;
  }
  __device__ __forceinline__ void start(const Item* r, uint64_t* f, volatile int* a) {
    ring = r;
    full = f;
    abort = a;
    ii = -1;
    next_item();
  }
  __device__ __forceinline__ void advance() {
    if (++c >= nchunks) next_item();
  }
};

// Q rows of a tile by TMA: box (64 elements of head_dim, g heads, 128 / g
// tokens) of the query tensor (head_dim, heads, tokens), 128B swizzle.
__device__ __forceinline__ void tma_load_q(void* dst, const CUtensorMap* map, int x, int y, int z,
                                           uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_q(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// 16 bytes global -> shared without registers; zeros when !valid.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

// QT: Q is copied by TMA (g divides 128, so a tile's rows are whole tokens);
// otherwise the softmax threads copy their rows.
// OT: query/output type. F8: the cache holds E4M3 codes, widened to f16 in
// shared memory by the producer and the widening warp; a bf16 Q is rounded to
// f16 (the MMAs are f16): in place by the tile's MMA warp when it came by TMA,
// by the softmax threads as they stage it otherwise.
template <typename OT, int D, bool QT, bool F8>
__global__ void __launch_bounds__(F8 ? kThreads8 : kThreads, 1)
    prefill_tc5_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v,
                       const __grid_constant__ CUtensorMap tmap_q, int num_seqs, int tiles,
                       int n_items, int* sched) {
  using T = typename std::conditional<F8, __half, OT>::type;  // MMA operand type
  using C = Cfg5<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;                          // C::kNSx stages: K pieces, V pieces
  uint8_t* ring8 = ring + C::kNSx * C::kStage;       // F8: C::kNS8x stages of E4M3 codes
  uint8_t* qs = ring8 + C::kNS8x * C::kStage8;       // Q pieces of tile 0, then of tile 1
  uint64_t* full = reinterpret_cast<uint64_t*>(qs + kTiles * C::kQ);
  uint64_t* empty = full + C::kNSx;
  uint64_t* s_full = empty + C::kNSx;         // [tile][buffer] S of a chunk is in tensor memory
  uint64_t* p_full = s_full + 2 * kTiles;  // [tile][buffer] P of a chunk is in tensor memory
  uint64_t* q_full = p_full + 2 * kTiles;  // [tile] Q of the tile's next item is staged
  uint64_t* o_done = q_full + kTiles;      // [tile] every PV of the tile's item has completed
  uint64_t* drain = o_done + kTiles;       // every MMA issued has completed
  uint64_t* full8 = drain + 1;               // F8: [kNS8x] E4M3 codes of a chunk have landed
  uint64_t* free8 = full8 + C::kNS8x;        // F8: [kNS8x] both halves of its chunk are widened
  uint32_t* tslot = reinterpret_cast<uint32_t*>(free8 + C::kNS8x);
  volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);
  uint64_t* item_full = reinterpret_cast<uint64_t*>(tslot + 2);  // [kRing] a record is published
  uint64_t* item_empty = item_full + kRing;  // [kRing] every role is done with a record
  Item* ring_items = reinterpret_cast<Item*>(item_empty + kRing);

  const int Hq = p.num_heads, g = Hq / p.num_kv_heads, bs = p.block_size;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kNSx; ++s) {
      // F8: every lane of the producer (K) and of the widening warp (V)
      mbar_init(full + s, F8 ? 64 : 1);
      mbar_init(empty + s, kTiles);  // one commit per tile's MMA warp
    }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(s_full + 2 * t, 1);
      mbar_init(s_full + 2 * t + 1, 1);
      mbar_init(p_full + 2 * t, kRows);
      mbar_init(p_full + 2 * t + 1, kRows);
      mbar_init(q_full + t, QT ? 1 : kRows);
      mbar_init(o_done + t, 1);
    }
    mbar_init(drain, kTiles);
    if (F8)
      for (int s = 0; s < C::kNS8x; ++s) {
        mbar_init(full8 + s, 1);
        mbar_init(free8 + s, 64);  // every lane of both widening warps
      }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(item_full + s, 1);
      mbar_init(item_empty + s, kTiles + kSoftWarps);  // the MMA warps and the softmax warps
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // F8: one tensor (0 = K, 1 = V) of a chunk's codes widened, exactly, to f16
  // in the chunk's 16-bit stage. Lane = (row a of each kRpi-row band, 16-byte
  // group jj of codes): the group, its 16-bit piece and both swizzles are fixed
  // per lane. All of the lane's codes are loaded before the first store: the
  // stores may alias the loads as far as the compiler knows, so loads left
  // between them would each wait out a shared-memory round trip (measured 2x
  // slower in isolation).
  auto widen_half = [&](const uint8_t* st8, uint8_t* st, int tensor) {
    constexpr int kGpr = D / 16, kRpi = 32 / kGpr;
    const int jj = lane % kGpr, a = lane / kGpr;
    const int pc = jj >> 2, g0 = 2 * (jj & 3);
    constexpr int kN = kChunk / kRpi;
    uint4 v[kN];
#pragma unroll
    for (int i = 0; i < kN; ++i) {
      const int r = a + kRpi * i;
      const int x8 = C::kRowB8 == 128 ? (r & 7) : ((r >> 1) & 3);
      v[i] = *reinterpret_cast<const uint4*>(st8 + tensor * C::kKV8 + r * C::kRowB8 +
                                             ((jj ^ x8) << 4));
    }
#pragma unroll
    for (int i = 0; i < kN; ++i) {
      const int r = a + kRpi * i;
      uint8_t* d = st + tensor * C::kKV + pc * C::kPlaneKV + r * 128;
      uint4 o0, o1;
      e4m3x4_to_f16x4(v[i].x, o0.x, o0.y);
      e4m3x4_to_f16x4(v[i].y, o0.z, o0.w);
      e4m3x4_to_f16x4(v[i].z, o1.x, o1.y);
      e4m3x4_to_f16x4(v[i].w, o1.z, o1.w);
      *reinterpret_cast<uint4*>(d + ((g0 ^ (r & 7)) << 4)) = o0;
      *reinterpret_cast<uint4*>(d + (((g0 + 1) ^ (r & 7)) << 4)) = o1;
    }
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer ----
    const int piece = bs * 128;  // bytes of one (block, piece of head_dim) box
    uint32_t armed = 0, last_parity = 0;
    bool ok = true;
    // Takes the next item of the launch (lane 0, from the work counter),
    // publishes its record (one with no chunks when the work is gone) and
    // starts its Q on the way into L2.
    int ii = -1;
    Item cur;
    auto publish = [&]() -> bool {
      ++ii;
      const int slot = ii % kRing;
      if (lane == 0) ok = wait5(item_empty + slot, ((uint32_t)(ii / kRing) & 1u) ^ 1u, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      if (lane == 0) {
        Item it;
        for (;;) {
          const int i = atomicAdd(sched, 1);
          if (i >= n_items) {
            it.nchunks = 0;
            break;
          }
          if (load_item(p, num_seqs, tiles, i, it)) break;
        }
        ring_items[slot] = it;
        mbar_arrive(item_full + slot);
        if (QT && it.nchunks > 0) {
#pragma unroll
          for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int pc = 0; pc < C::kPlanes; ++pc)
              tma_prefetch_q(&tmap_q, pc * 64, it.h * g, it.q0 + (it.row0 + kRows * t) / g);
        }
      }
      __syncwarp();
      cur = ring_items[slot];
      if (!QT && cur.nchunks > 0) {  // its Q rows into L2 (the softmax threads copy them)
        for (int rr = lane; rr < kCtaRows; rr += 32) {
          const int R = cur.row0 + rr;
          if (R >= cur.rows) break;
          const int tk = R / g;
          const char* qr = reinterpret_cast<const char*>(
              static_cast<const OT*>(p.query) + ((int64_t)(cur.q0 + tk) * Hq + cur.h * g +
                                                 (R - tk * g)) * D);
#pragma unroll
          for (int b = 0; b < D * (int)sizeof(OT); b += 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(qr + b));
        }
      }
      return cur.nchunks > 0;
    };
    if constexpr (F8) {
      // E4M3 cache: TMA copies of a chunk's codes into the staging ring run one
      // chunk ahead of their widening (exact) to f16 in the chunk's stage, in
      // the same layout the 16-bit path gets from TMA; then the stage is full.
      const int piece8 = bs * C::kRowB8;  // bytes of one (block) box of codes
      uint32_t armed8 = 0, last8 = 0;
      int lc = 0, lj = 0;  // load cursor: chunk within `cur`, chunk index
      bool lhave = publish();
      auto issue_load = [&]() {
        const int s8 = lj % C::kNS8x;
        // Both halves of the slot's previous chunk have been widened.
        ok = wait5(free8 + s8, ((uint32_t)(lj / C::kNS8x) & 1u) ^ 1u, abort);
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          return;
        }
        const int c0 = lc * kChunk;
        const int nblk = (min(kChunk, cur.kv_end - c0) + bs - 1) / bs;
        const int32_t* bt = p.block_table + (int64_t)cur.seq * p.max_blocks_per_seq;
        const int blk = lane < nblk ? __ldg(bt + c0 / bs + lane) : 0;
        uint8_t* st8 = ring8 + s8 * C::kStage8;
        if (lane == 0) mbar_expect_tx(full8 + s8, (uint32_t)(2 * nblk * piece8));
        __syncwarp();
        if (lane < nblk) {
          if (blk < 0 || blk >= p.num_blocks) atomicOr(&g_pf5_status, 2);  // reads as zeros
          tma_load_5d(st8 + lane * piece8, &tmap_k, 0, 0, 0, cur.h, blk, full8 + s8);
          tma_load_5d(st8 + C::kKV8 + lane * piece8, &tmap_v, 0, 0, 0, cur.h, blk, full8 + s8);
        }
        armed8 |= 1u << s8;
        last8 = (last8 & ~(1u << s8)) | (((uint32_t)(lj / C::kNS8x) & 1u) << s8);
        ++lj;
        if (++lc >= cur.nchunks) {
          lc = 0;
          lhave = publish();
        }
      };
      for (int k = 0; k < C::kNS8x - 1 && lhave && ok; ++k) issue_load();
      int ci = 0, cc = 0;  // the widening cursor: item number in the ring, chunk within it
      for (int j = 0; ok; ++j) {
        const int nch = ring_items[ci % kRing].nchunks;  // published by the load cursor
        if (nch == 0) break;                              // the work is gone
        if (lhave) issue_load();  // chunk j + kNS8x - 1, into the slot chunk j - 1 left
        if (!ok) break;
        const int stage = j % C::kNSx;
        // Every lane waits, widens, fences its own stores and arrives: with a
        // wait in one lane and a warp sync before the arrival, the warp ran
        // the widening as two groups of lanes, one after the other (measured).
        ok = wait5(empty + stage, ((uint32_t)(j / C::kNSx) & 1u) ^ 1u, abort);
        if (ok) ok = wait5(full8 + j % C::kNS8x, (uint32_t)(j / C::kNS8x) & 1u, abort);
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          break;
        }
        const uint8_t* st8 = ring8 + (j % C::kNS8x) * C::kStage8;
        uint8_t* st = ring + stage * C::kStage;
        widen_half(st8, st, 0);  // K (the widening warp does V)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // for the tensor cores
        mbar_arrive(full + stage);
        mbar_arrive(free8 + j % C::kNS8x);
        if (++cc >= nch) {
          cc = 0;
          ++ci;
        }
      }
      if (!ok && lane == 0) {  // wait, bounded, for this CTA's copies in flight
        for (int s8 = 0; s8 < C::kNS8x; ++s8) {
          if (!(armed8 >> s8 & 1u)) continue;
          const long long t0 = clock64();
          while (!mbar_try(full8 + s8, (last8 >> s8) & 1u))
            if (clock64() - t0 > kWaitCycles) break;
        }
      }
    } else {
    bool have = publish();
    for (int j = 0, c = 0; have && ok; ++j) {
      const int stage = j % C::kNSx;
      const uint32_t phase = (uint32_t)(j / C::kNSx) & 1u;
      const int c0 = c * kChunk;
      const int nblk = (min(kChunk, cur.kv_end - c0) + bs - 1) / bs;
      const int32_t* bt = p.block_table + (int64_t)cur.seq * p.max_blocks_per_seq;
      const int blk = lane < nblk ? __ldg(bt + c0 / bs + lane) : 0;
      if (lane == 0) ok = wait5(empty + stage, phase ^ 1u, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* st = ring + stage * C::kStage;
      if (lane == 0) mbar_expect_tx(full + stage, (uint32_t)(2 * C::kPlanes * nblk * piece));
      __syncwarp();
      if (lane < nblk) {
        if (blk < 0 || blk >= p.num_blocks) atomicOr(&g_pf5_status, 2);  // reads as zeros
#pragma unroll
        for (int pc = 0; pc < C::kPlanes; ++pc) {
          tma_load_5d(st + pc * C::kPlaneKV + lane * piece, &tmap_k, 0, 0, pc, cur.h, blk,
                      full + stage);
          tma_load_5d(st + C::kKV + pc * C::kPlaneKV + lane * piece, &tmap_v, 0, 0, pc, cur.h,
                      blk, full + stage);
        }
      }
      armed |= 1u << stage;
      last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
      if (++c >= cur.nchunks) {
        c = 0;
        have = publish();
      }
    }
    if (!ok && lane == 0) {  // wait, bounded, for this CTA's copies in flight
      for (int s = 0; s < C::kNSx; ++s) {
        if (!(armed >> s & 1u)) continue;
        const long long t0 = clock64();
        while (!mbar_try(full + s, (last_parity >> s) & 1u))
          if (clock64() - t0 > kWaitCycles) break;
      }
    }
    }  // 16-bit cache
  } else if (warp == kWidenWarp) {  // only launched with an E4M3 cache
    // ------------------------------------------------------ V widening (F8) ----
    if constexpr (F8) {
    Walk w;
    w.start(ring_items, item_full, abort);
    bool ok = true;
    for (int j = 0; w.ok && ok; ++j) {
      const int stage = j % C::kNSx;
      // As in the producer, every lane waits, widens and arrives.
      ok = wait5(empty + stage, ((uint32_t)(j / C::kNSx) & 1u) ^ 1u, abort);
      if (ok) ok = wait5(full8 + j % C::kNS8x, (uint32_t)(j / C::kNS8x) & 1u, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      widen_half(ring8 + (j % C::kNS8x) * C::kStage8, ring + stage * C::kStage, 1);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // for the tensor cores
      mbar_arrive(full + stage);
      mbar_arrive(free8 + j % C::kNS8x);
      w.advance();
    }
    }
  } else if (warp >= kMmaWarp && warp < kMmaWarp + kTiles) {
    // ----------------------------------------------------------------- MMA ----
    // Warp kMmaWarp + t serves tile t over the chunk sequence of all this
    // CTA's items: S of chunks 0 and 1 up front (one S buffer each), then per
    // chunk j: O_t += P_t(j) V(j) once the tile's softmax has written P(j)
    // over its S buffer, then S_t(j + 2) into that buffer (of the next item
    // when j + 2 is past this one's end: its Q is waited for first), while
    // S(j + 1), in the other buffer, was computed during the softmax of chunk
    // j. Past the last chunk a commit alone stands in for S(j + 2). The whole
    // warp runs the loop on warp-uniform operands; one elected thread issues.
    constexpr uint32_t idS = idesc<T>(kRows, kChunk, false);
    constexpr uint32_t idO = idesc<T>(kRows, D, true);
    const uint32_t q_addr = smem_u32(qs), r_addr = smem_u32(ring);
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const bool leader = elect_one();
    const int t = warp - kMmaWarp;  // this warp issues the MMAs of tile t
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, wait5(bar, parity, abort));
    };
    auto issue_s = [&](int j) {  // S_t(j) = Q_t K(j)^T into buffer j % 2
      // Base descriptors once; the K steps add compile-time offsets to the
      // 14-bit address field (addresses stay below 256 KB, so it never carries).
      const uint64_t a0 = sdesc(q_addr + t * C::kQ, 16);
      const uint64_t b0 = sdesc(r_addr + (j % C::kNSx) * C::kStage, 16);
      const uint32_t dS = tm + 128 * t + 64 * (j & 1);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const int pc = s / 4, off = (s % 4) * 32;
        umma(dS, a0 + (uint64_t)((pc * C::kPlaneQ + off) >> 4),
             b0 + (uint64_t)((pc * C::kPlaneKV + off) >> 4), idS, s > 0 ? 1u : 0u);
      }
      umma_commit(s_full + 2 * t + (j & 1));
    };
    auto issue_pv = [&](int j, bool acc) {  // O_t (+)= P_t(j) V(j)
      const uint64_t b0 = sdesc(r_addr + (j % C::kNSx) * C::kStage + C::kKV, C::kPlaneKV);
      const uint32_t dO = tm + C::kColO + t * D, aP = tm + 128 * t + 64 * (j & 1);
#pragma unroll
      for (int s = 0; s < kChunk / 16; ++s)
        umma_ts(dO, aP + 8 * s, b0 + (uint64_t)((s * 16 * 128) >> 4), idO,
                (acc || s > 0) ? 1u : 0u);
    };
    Walk pv, sn;  // the chunk of the next PV, and of the next S (two ahead)
    pv.start(ring_items, item_full, abort);
    sn.start(ring_items, item_full, abort);
    int js = 0, q_items = 0;
    auto next_s = [&]() -> bool {
      if (!sn.ok) {  // past the last chunk
        if (leader) umma_commit(s_full + 2 * t + (js & 1));
        __syncwarp();
        ++js;
        return true;
      }
      if (sn.c == 0) {  // the first S of an item: its Q must be staged
        if (!wait_warp(q_full + t, (uint32_t)q_items & 1u)) return false;
        ++q_items;
        if constexpr (F8 && QT && !std::is_same<OT, __half>::value) {
          // The tile's Q came by TMA as bf16: rounded to f16 in place for the
          // f16 MMAs (every 16-bit element on its own, so the swizzle does not
          // matter); each lane fences its stores before the warp sync.
          uint4* qb = reinterpret_cast<uint4*>(qs + t * C::kQ);
#pragma unroll 4
          for (int e = lane; e < C::kQ / 16; e += 32) {
            const uint4 v = qb[e];
            qb[e] = make_uint4(to_f16x2<OT>(v.x), to_f16x2<OT>(v.y), to_f16x2<OT>(v.z),
                               to_f16x2<OT>(v.w));
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
      }
      // K of chunk js (waited for only now, so the PV before never waits on a copy).
      if (!wait_warp(full + js % C::kNSx, (uint32_t)(js / C::kNSx) & 1u)) return false;
      tc_fence_after();
      if (leader) issue_s(js);
      __syncwarp();
      ++js;
      sn.advance();
      return true;
    };
    bool ok = !pv.ok || (next_s() && next_s());
    for (int j = 0; pv.ok && ok; ++j) {
      ok = wait_warp(p_full + 2 * t + (j & 1), (uint32_t)(j >> 1) & 1u);
      if (!ok) break;
      tc_fence_after();
      const bool last = pv.c == pv.nchunks - 1;
      if (leader) {
        issue_pv(j, pv.c > 0);
        umma_commit(empty + j % C::kNSx);
        if (last) umma_commit(o_done + t);
      }
      __syncwarp();
      ok = next_s();
      if (last && lane == 0) mbar_arrive(item_empty + pv.ii % kRing);  // done with its record
      pv.advance();
    }
    // Whatever happened, wait (bounded) until every MMA issued has completed.
    if (leader) {
      umma_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try(drain, 0))
        if (clock64() - t0 > kWaitCycles) break;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax ----
    const int t = warp / 4;                 // this warp's tile
    const int r = 32 * (warp % 4) + lane;   // this thread's tensor-memory lane and row of the tile
    const uint32_t trow = tmem + ((uint32_t)(32 * (warp % 4)) << 16);
    const uint32_t tO = trow + C::kColO + t * D;
    const uint32_t qt = smem_u32(qs + t * C::kQ);
    // This thread's row of Q of an item (zeros past its rows), copied into the
    // operand layout without passing through registers; q_ready() publishes it.
    auto stage_q = [&](const Item& it) {
      const int R = it.row0 + kRows * t + r;
      const bool valid = R < it.rows;
      const int tok = valid ? R / g : 0, jh = valid ? R - tok * g : 0;
      const uint4* src = reinterpret_cast<const uint4*>(
          static_cast<const OT*>(p.query) + ((int64_t)(it.q0 + tok) * Hq + it.h * g + jh) * D);
      if constexpr (F8 && !std::is_same<OT, __half>::value) {
        // The f16 MMAs of an E4M3 cache: Q rounded to f16 on its way in.
        uint4 v[D / 8];
#pragma unroll
        for (int u = 0; u < D / 8; ++u) v[u] = valid ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
          uint4 h;
          h.x = to_f16x2<OT>(v[u].x);
          h.y = to_f16x2<OT>(v[u].y);
          h.z = to_f16x2<OT>(v[u].z);
          h.w = to_f16x2<OT>(v[u].w);
          *reinterpret_cast<uint4*>(qs + t * C::kQ + (u >> 3) * C::kPlaneQ + sw(r, u & 7)) = h;
        }
      } else {
#pragma unroll
        for (int u = 0; u < D / 8; ++u)
          cp_async16(qt + (u >> 3) * C::kPlaneQ + sw(r, u & 7), valid ? src + u : p.query, valid);
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
    };
    auto q_ready = [&]() {
      asm volatile("cp.async.wait_all;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(q_full + t);
    };
    // With TMA one thread of the tile loads (or prefetches into L2) an item's Q.
    const bool q_thread = r == 0;
    int q_loads = 0;  // Q copies this thread has issued
    auto load_q_tma = [&](const Item& it) {
      ++q_loads;
      const int z = it.q0 + (it.row0 + kRows * t) / g;
      mbar_expect_tx(q_full + t, (uint32_t)C::kQ);
#pragma unroll
      for (int pc = 0; pc < C::kPlanes; ++pc)
        tma_load_q(qs + t * C::kQ + pc * C::kPlaneQ, &tmap_q, pc * 64, it.h * g, z, q_full + t);
    };
    // E4M3: K = code * k_scale folds into the score scale, V = code * v_scale
    // into the output.
    const float sscale = p.score_scale * (F8 ? __ldg(p.k_scale) : 1.f);
    const float vsc = F8 ? __ldg(p.v_scale) : 1.f;
    Walk w;
    w.start(ring_items, item_full, abort);
    if (w.ok) {
      if (QT) {
        if (q_thread) load_q_tma(w.it());
      } else {
        stage_q(w.it());
        q_ready();
      }
    }
    bool ok = true;
    int j = 0, items = 0;
    // The previous item's O is read and stored (its epilogue) only after the
    // next item's first chunk has been through the softmax and before that
    // chunk's P is published: the wait for the previous item's last PV then
    // overlaps useful work, and the next item's first PV, which overwrites O,
    // cannot start before O has been read.
    bool pending = false, prev_valid = false;
    // Output rows are D * 2 bytes: all 32-byte aligned when the output is.
    const bool out32 = !F8 && (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
    uint64_t prev_lsum = 0;
    OT* prev_dst = nullptr;
    auto epilogue = [&]() -> bool {
      pending = false;
      bool okk = wait5(o_done + t, (uint32_t)items & 1u, abort);  // every PV of the item
      okk = __all_sync(0xffffffffu, okk);
      ++items;
      if (!okk) return false;
      tc_fence_after();
      float l0, l1;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(l0), "=f"(l1) : "l"(prev_lsum));
      const float lsum = l0 + l1;
      const float inv = lsum > 0.f ? vsc / lsum : 0.f;
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        float o[64];
        tmem_ld64(tO + 64 * q, o);  // two loads in flight, one wait
        if (!F8 && prev_valid && out32) {
          // 16-bit caches: 32 bytes (a whole sector) per store when the output
          // is 32-byte aligned; sixteen-byte stores left each sector half
          // written by two instructions (the E4M3 form keeps them: measured
          // faster there)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t wv[8];
            float a, b;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              wv[k] = Mma<OT>::pack(o[16 * u + 2 * k] * inv, o[16 * u + 2 * k + 1] * inv, a, b);
            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                             prev_dst + 64 * q + 16 * u),
                         "r"(wv[0]), "r"(wv[1]), "r"(wv[2]), "r"(wv[3]), "r"(wv[4]), "r"(wv[5]),
                         "r"(wv[6]), "r"(wv[7])
                         : "memory");
          }
        } else if (prev_valid) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 wv;
            float a, b;
            wv.x = Mma<OT>::pack(o[8 * u + 0] * inv, o[8 * u + 1] * inv, a, b);
            wv.y = Mma<OT>::pack(o[8 * u + 2] * inv, o[8 * u + 3] * inv, a, b);
            wv.z = Mma<OT>::pack(o[8 * u + 4] * inv, o[8 * u + 5] * inv, a, b);
            wv.w = Mma<OT>::pack(o[8 * u + 6] * inv, o[8 * u + 7] * inv, a, b);
            *reinterpret_cast<uint4*>(prev_dst + 64 * q + 8 * u) = wv;
          }
        }
      }
      return true;
    };
    while (w.ok && ok) {
      const int nchunks = w.it().nchunks, kv_end = w.it().kv_end;
      const int R = w.it().row0 + kRows * t + r;
      const bool valid = R < w.it().rows;
      const int tok = valid ? R / g : 0, jh = valid ? R - tok * g : 0;
      const int pos = valid ? w.it().base_pos + tok : -1;
      OT* const dst =
          static_cast<OT*>(p.out) + ((int64_t)(w.it().q0 + tok) * Hq + w.it().h * g + jh) * D;
      __syncwarp();  // every lane has read the record
      if (lane == 0) mbar_arrive(item_empty + w.ii % kRing);
      float m_use = -INFINITY;
      uint64_t lsum2 = 0;
      bool q_pending = false;
      for (int c = 0; c < nchunks; ++c, ++j) {
        ok = wait5(s_full + 2 * t + (j & 1), (uint32_t)(j >> 1) & 1u, abort);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (c == nchunks - 1) w.next_item();  // w is the next item from here on
        if (c == nchunks - 1 && w.ok) {
          // Every S of this item has completed (this is its last), so Q's
          // buffer is free: fetch the next item's rows while this chunk and
          // the epilogue run.
          if (QT) {
            if (q_thread) load_q_tma(w.it());
          } else {
            stage_q(w.it());
            q_pending = true;
          }
        }
        const uint32_t tS = trow + 128 * t + 64 * (j & 1);
        float s[64];
        tmem_ld64(tS, s);
        const int c0 = c * kChunk;
        // Raw scores; the causal mask only where the chunk reaches past a row's
        // position. The scale is applied with the exponent (it is positive, so the
        // maximum of the raw scores gives the maximum of the scaled ones).
        if (__any_sync(0xffffffffu, c0 + kChunk - 1 > pos)) {
#pragma unroll
          for (int i = 0; i < 64; ++i) s[i] = c0 + i <= pos ? s[i] : -INFINITY;
        }
        const float mx = max64(s) * sscale;
        // Raise the running maximum only when this chunk exceeds it by 2^8.
        const bool raise = mx > m_use + 8.f;
        const bool rescale = raise && m_use != -INFINITY;
        // The PV of the previous chunk must have completed before O is rescaled:
        // the commit of S(j + 1) (or of its stand-in) follows it. At an item's
        // last chunk S(j + 1) is the next item's first, which needs its Q.
        if (__any_sync(0xffffffffu, rescale)) {
          if (c > 0) {
            if (q_pending) {
              q_ready();
              q_pending = false;
            }
            ok = wait5(s_full + 2 * t + ((j + 1) & 1), (uint32_t)((j + 1) >> 1) & 1u, abort);
            if (!__all_sync(0xffffffffu, ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const float alpha = rescale ? fast_exp2(m_use - mx) : 1.f;
          {
            uint64_t aa;
            asm("mov.b64 %0, {%1, %1};" : "=l"(aa) : "f"(alpha));
            asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(lsum2) : "l"(aa));
          }
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            float o[32];
            tmem_ld32(tO + 32 * q, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + 32 * q, o);
          }
        }
        if (raise) m_use = mx;
        const float msub = m_use == -INFINITY ? 0.f : m_use;
        uint32_t pk[32];
        float ls0, ls1;  // the two halves of the row sums, for the 16-bit adds below
        asm("mov.b64 {%0, %1}, %2;" : "=f"(ls0), "=f"(ls1) : "l"(lsum2));
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float x0, x1;  // s * scale - m for a pair, as one packed f32x2 FMA
          {
            uint64_t xy, sc, mm, rr;
            asm("mov.b64 %0, {%1, %2};" : "=l"(xy) : "f"(s[2 * i]), "f"(s[2 * i + 1]));
            asm("mov.b64 %0, {%1, %1};" : "=l"(sc) : "f"(sscale));
            asm("mov.b64 %0, {%1, %1};" : "=l"(mm) : "f"(-msub));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rr) : "l"(xy), "l"(sc), "l"(mm));
            asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(rr));
          }
          float lo, hi;  // the row sums take P as the tensor cores see it (bf16: rounded)
          if constexpr (F8) {
            // f16 P is within 2^-11 (relative) of the fp32 value, and reading
            // it back would cost two conversions per pair: the row sums take
            // the fp32 values.
            lo = fast_exp2(x0);
            hi = fast_exp2(x1);
            const __half2 hv = __floats2half2_rn(lo, hi);
            pk[i] = *reinterpret_cast<const uint32_t*>(&hv);
          } else {
            pk[i] = Mma<T>::pack(fast_exp2(x0), fast_exp2(x1), lo, hi);
          }
          if constexpr (F8) {
            uint64_t pp;
            asm("mov.b64 %0, {%1, %2};" : "=l"(pp) : "f"(lo), "f"(hi));
            asm("add.rn.f32x2 %0, %0, %1;" : "+l"(lsum2) : "l"(pp));
          } else {
            // The rounded pair added to the sums as it is: each 16-bit value is
            // converted exactly and added in fp32 by one instruction (sm_100's
            // mixed-precision add), where unpacking the pair first took three.
            (void)lo;
            (void)hi;
            if constexpr (std::is_same<T, __nv_bfloat16>::value)
              asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n add.rn.f32.bf16 %0, l, %0;\n"
                  " add.rn.f32.bf16 %1, h, %1;\n}" : "+f"(ls0), "+f"(ls1) : "r"(pk[i]));
            else
              asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n add.rn.f32.f16 %0, l, %0;\n"
                  " add.rn.f32.f16 %1, h, %1;\n}" : "+f"(ls0), "+f"(ls1) : "r"(pk[i]));
          }
        }
        if constexpr (!F8) asm("mov.b64 %0, {%1, %2};" : "=l"(lsum2) : "f"(ls0), "f"(ls1));
        if (c == nchunks - 1 && c0 + kChunk > kv_end) {
          // Zero V rows past the range (stale or poisoned) before this tile's
          // last PV. Both tiles do it, as their PVs are issued independently
          // (the other tile's stores write the same zeros).
          uint8_t* v = ring + (j % C::kNSx) * C::kStage + C::kKV;
          const int t0 = kv_end - c0, per_row = 8 * C::kPlanes;
          for (int e = r; e < (kChunk - t0) * per_row; e += kRows) {
            const int tk = t0 + e / per_row, u = e % per_row;
            *reinterpret_cast<uint4*>(v + (u >> 3) * C::kPlaneKV + tk * 128 + (u & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        // P over the first 32 columns of this chunk's S buffer (S is in registers).
        tmem_st32(tS, pk);
        if (c == 0 && pending && !epilogue()) {
          ok = false;
          break;
        }
        tc_fence_before();
        mbar_arrive(p_full + 2 * t + (j & 1));
        if (q_pending) {
          q_ready();
          q_pending = false;
        }
      }
      if (!ok) break;
      // This item's epilogue waits until the next item's first chunk has been
      // through the softmax (or until the end).
      prev_lsum = lsum2;
      prev_dst = dst;
      prev_valid = valid;
      pending = true;
    }
    if (ok && pending) ok = epilogue();
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing left in flight on any path
    if (QT && q_thread && q_loads > 0) {  // nor a Q copy (an aborted call may not have used it)
      const long long t0 = clock64();
      while (!mbar_try(q_full + t, (uint32_t)(q_loads - 1) & 1u))
        if (clock64() - t0 > kWaitCycles) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
  if (threadIdx.x == 0) {  // the last CTA of the launch leaves the work counter at 0
    __threadfence();
    if (atomicAdd(sched + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(sched, 0);
      atomicExch(sched + 1, 0);
    }
  }
}

// The work counter of the next launch: each launch takes the next of
// kSchedSlots (the last CTA of a launch resets its slot), so up to kSchedSlots
// calls may be in flight at once, on any streams.
cudaError_t next_sched_slot(int dev, int** sched) {
  static std::atomic<unsigned> launches{0};
  static std::atomic<int*> base[64];
  int* b = base[dev].load(std::memory_order_relaxed);
  if (!b) {
    void* a = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&a, g_pf5_sched);
    if (e != cudaSuccess) return e;
    b = static_cast<int*>(a);
    base[dev].store(b, std::memory_order_relaxed);
  }
  *sched = b + 2 * (int)(launches.fetch_add(1, std::memory_order_relaxed) % kSchedSlots);
  return cudaSuccess;
}

template <typename OT, int D, bool QT, bool F8>
cudaError_t launch5(const PrefillParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mq, int num_seqs, cudaStream_t stream) {
  using C = Cfg5<D, F8>;
  auto kernel = prefill_tc5_kernel<OT, D, QT, F8>;
  static std::atomic<int> opted_in[64];  // the shared-memory opt-in, once per device
  static std::atomic<int> sm_count[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!opted_in[dev].load(std::memory_order_relaxed)) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sm_count[dev].store(n > 0 ? n : 1, std::memory_order_relaxed);
    opted_in[dev].store(1, std::memory_order_relaxed);
  }
  const int g = p.num_heads / p.num_kv_heads;
  const int64_t tiles = ((int64_t)p.max_q_len * g + kCtaRows - 1) / kCtaRows;
  const int64_t n_items = tiles * num_seqs * p.num_kv_heads;
  if (n_items <= 0) return cudaSuccess;
  if (n_items > (int64_t)INT32_MAX / 2) return cudaErrorInvalidValue;
  // Persistent: one CTA per SM (a CTA fills one), each taking the launch's
  // items from a work counter as it becomes free.
  int* sched = nullptr;
  const cudaError_t es = next_sched_slot(dev, &sched);
  if (es != cudaSuccess) return es;
  const int64_t grid = std::min<int64_t>(n_items, sm_count[dev].load(std::memory_order_relaxed));
  kernel<<<(unsigned)grid, F8 ? kThreads8 : kThreads, C::kSmem, stream>>>(p, mk, mv, mq, num_seqs, (int)tiles,
                                                         (int)n_items, sched);
  return cudaGetLastError();
}

// The query tensor (head_dim, heads, tokens) for Q tiles by TMA: box (64, g,
// 128 / g) in the 128B swizzle. False when g does not divide 128.
bool encode_q_map(CUtensorMap* map, const PrefillParams& p, int head_dim, bool bf16) {
  const int g = p.num_heads / p.num_kv_heads;
  if (kRows % g != 0) return false;
  auto enc = tcx::tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)p.num_heads,
                        (cuuint64_t)p.num_q_tokens};
  cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)p.num_heads * head_dim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)(kRows / g)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(p.query), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename OT, int D>
cudaError_t launch5q(const PrefillParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                     bool f8, int num_seqs, cudaStream_t stream) {
  CUtensorMap mq;
  const bool qt = encode_q_map(&mq, p, D, std::is_same<OT, __nv_bfloat16>::value);
  if (f8)  // a bf16 Q is rounded to f16, in place, for the f16 MMAs
    return qt ? launch5<OT, D, true, true>(p, mk, mv, mq, num_seqs, stream)
              : launch5<OT, D, false, true>(p, mk, mv, mk, num_seqs, stream);  // mk: no Q map
  if (qt) return launch5<OT, D, true, false>(p, mk, mv, mq, num_seqs, stream);
  return launch5<OT, D, false, false>(p, mk, mv, mk, num_seqs, stream);  // mk unused as Q map
}

}  // namespace

bool prefill_tc5_supported(int head_dim) { return head_dim == 64 || head_dim == 128; }

cudaError_t launch_prefill_tc5(const PrefillParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                               int head_dim, bool bf16, bool f8, int num_seqs,
                               cudaStream_t stream) {
  if (bf16)
    return head_dim == 128 ? launch5q<__nv_bfloat16, 128>(p, mk, mv, f8, num_seqs, stream)
                           : launch5q<__nv_bfloat16, 64>(p, mk, mv, f8, num_seqs, stream);
  return head_dim == 128 ? launch5q<__half, 128>(p, mk, mv, f8, num_seqs, stream)
                         : launch5q<__half, 64>(p, mk, mv, f8, num_seqs, stream);
}

}  // namespace pf

int pf5_status_flag(bool clear, int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_pf5_status, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_pf5_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  *value = v;
  return 0;
}

}  // namespace pkv
