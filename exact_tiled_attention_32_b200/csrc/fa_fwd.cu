// fa_fwd.cu -- exact attention forward for B200 (sm_100a) and its C ABI.
//
// The method (pages: "Flash Attention", 14cs17.netlify.app -- "Tiling
// Strategy", "Online Softmax" (Theorem 2), "Flash Attention Algorithm",
// "Flash Attention 2 Improvements"): for each block Q_i of query rows, stream
// the key/value blocks K_j, V_j through on-chip memory, form S_ij = Q_i K_j^T,
// fold it into a running row maximum m, a running row sum l and an
// unnormalised output O, and write only O / l (and the logsumexp) to HBM.
//
// B200 mapping (one persistent CTA per SM, 384 threads, warp-specialised):
//   warps 0-3   query tile 0, warps 4-7 query tile 1 (one warpgroup each):
//               one thread per query row; tcgen05.ld of S, masking, running
//               max in the log2 domain, exp2 via one FFMA + ex2 (some column
//               pairs on an FMA-pipe polynomial at d = 64), lazy rescale of O
//               in TMEM (only when the max grows by more than 2^8), bf16 P
//               written to TMEM, and the epilogue O / l -> bf16 -> HBM plus
//               the logsumexp.
//   warp 10     MMA issuer: S_t = Q_t K_j^T as tcgen05.mma kind::f16 (bf16 in,
//               fp32 accumulate in TMEM); with the shared-S layout (bf16) it
//               issues only these, as soon as the shared S buffer is free.
//   warp 9      TMEM allocation; with the shared-S layout, the second MMA
//               issuer: O_t += P_t V_j with P read from TMEM, as soon as P_t
//               is written.  (FP8: warp 10 issues both kinds, in an order
//               that keeps the two softmax warpgroups out of phase.)
//   warp 11     TMA producer: Q (two 128-row tiles per work item) and a ring of
//               K_j / V_j tiles in 128-byte-swizzled shared memory.
//   warp 8      idle; it completes the third warpgroup, which gives registers
//               to the softmax warpgroups through setmaxnreg.
//
// TMEM (512 columns): see TmemLayout below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

namespace fa_sm100 {

constexpr int kBlockM = 128;           // query rows per tile (B_r)
constexpr int kBlockN = 128;           // keys per tile (B_c)
constexpr int kRowsPerItem = 2 * kBlockM;
constexpr int kNumSoftmaxWarps = 8;
constexpr int kAllocWarp = 9;
constexpr int kMmaWarp = 10;
constexpr int kLoadWarp = 11;
constexpr int kThreads = 384;
constexpr uint32_t kSoftmaxRegs = 216;   // setmaxnreg split: 2 x 128 x 216 + 128 x 72 = 384 x 168
constexpr uint32_t kOtherRegs = 72;
constexpr int kMaxSeqs = 1024;         // packed batches: sequences
constexpr int kMaxPairs = 1024;        // packed batches: 256-row pairs per sequence
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 10;
constexpr int kBoxBytes = kBlockM * 64 * 2;   // one 128-row x 64-column bf16 TMA box
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only past 2^8
// FP8: P is computed as 2^kF8Shift * exp2(x - m_used) and must stay within
// E4M3's largest value (448 = 2^8.807): with the reference m_used at most
// kF8Threshold below the row's true maximum, P <= 2^(kF8Shift + kF8Threshold).
#ifndef FA_F8_THRESHOLD
#define FA_F8_THRESHOLD 3.0f
#endif
constexpr float kF8Threshold = FA_F8_THRESHOLD;
constexpr float kF8Shift = FA_F8_THRESHOLD > 0.f ? 8.75f - FA_F8_THRESHOLD : 8.0f;
static_assert(kF8Shift + kF8Threshold <= 8.8f, "FP8 P must stay below 448");

// TMEM layouts (512 columns), per path:
//  kAlias   S0/P0 [0,128), S1/P1 [128,256), O0 [256,384), O1 [384,512):
//           P_t is written over S_t, so S_t(j+1) can only be computed after
//           P_t(j) V_j has read P_t(j): each tile's chain is softmax(j) ->
//           P V(j) -> S(j+1) -> softmax(j+1).
//  kSepP    (d = 64) S0 [0,128), S1 [128,256), P0 [256,320), P1 [320,384),
//           O0 [384,448), O1 [448,512): S_t(j+1) is computed as soon as the
//           softmax warps have loaded S_t(j) into registers.
//  kSharedS (d = 128) S [0,128) shared by both tiles, P0 [128,192),
//           P1 [192,256), O0 [256,384), O1 [384,512): the two tiles' scores
//           pass through one buffer in turn (S_0(j), S_1(j), S_0(j+1), ...),
//           each computed once the other tile's softmax warps have loaded
//           theirs, with the P V products of the tiles in between.
// In kSepP and kSharedS the softmax of block j+1 starts as soon as that of
// block j ends; the tensor core runs the other tile's work meanwhile.
enum TmemLayout : int { kAlias = 0, kSepP = 1, kSharedS = 2 };
#ifndef FA_LAYOUT_D64
#define FA_LAYOUT_D64 2
#endif
#ifndef FA_LAYOUT_D128
#define FA_LAYOUT_D128 2
#endif
#ifndef FA_LAYOUT_F8
#define FA_LAYOUT_F8 0
#endif
template <int D, bool F8>
__host__ __device__ constexpr int tmem_layout() {
    return F8 ? FA_LAYOUT_F8 : (D == 64 ? FA_LAYOUT_D64 : FA_LAYOUT_D128);
}

template <int D, bool F8>
__host__ __device__ constexpr bool sep_p() {
    return tmem_layout<D, F8>() != kAlias;
}
template <int D, bool F8>
__host__ __device__ constexpr uint32_t tmem_s_col(int t) {
    return tmem_layout<D, F8>() == kSharedS ? 0u : 128u * t;
}
template <int D, bool F8>
__host__ __device__ constexpr uint32_t tmem_p_col(int t) {
    return tmem_layout<D, F8>() == kSepP ? 256u + 64u * t
                                         : (tmem_layout<D, F8>() == kSharedS ? 128u + 64u * t : 128u * t);
}
template <int D, bool F8>
__host__ __device__ constexpr uint32_t tmem_o_col(int t) {
    return tmem_layout<D, F8>() == kSepP ? 384u + 64u * t : 256u + 128u * t;
}
static_assert(tmem_o_col<64, false>(1) + 64 <= 512 && tmem_o_col<128, false>(1) + 128 <= 512, "TMEM columns");

// where a wait gave up (reported in status[1])
enum WaitSite : int {
    kSiteQEmpty = 1, kSiteKvEmpty, kSiteQFull, kSiteKvFull, kSitePFull, kSiteSFull, kSiteOFinal, kSiteSFree,
    kSitePvDone, kSiteFeed
};

struct alignas(64) Params {
    CUtensorMap tm_q, tm_k, tm_v;
    void* o;
    float* lse;
    const int32_t* cu_seqlens;
    const int32_t* cu_seqlens_k;   // packed query chunks: key offsets (NULL: the keys are the queries' tokens)
    int* status;
    unsigned long long* sched;   // work counter: {launch epoch (bits 32-63), items taken (0-31)}
    unsigned epoch;              // this launch's epoch (nonzero)
    int dyn;                     // 1: dynamic schedule (sched, epoch); 0: static snake
    int B, Hq, Hkv, N;         // N: query rows per sequence (dense) or total tokens (packed)
    int Nk;                    // dense: keys per sequence (== N except for a query chunk)
    int q_off;                 // dense: position of query row 0 among the keys (Nk - N for a chunk)
    int qmod;                  // dense: row r sits at position q_off + r % qmod (rows of several
                               // query heads packed into one sequence); 0: position q_off + r
    int splits;                // dense: key blocks of each tile are cut into this many splits
    float* o_part;             // dense, when set: fp32 O / l of each split, [splits][B*Hq*N][d]
    float* lse_part;           // dense, when set: logsumexp of each split, [splits][B*Hq*N]
    int group;                 // Hq / Hkv
    int group_units;           // dense: (batch, head) units scheduled together
    long long l2_group_bytes;  // packed, dynamic schedule: K/V bytes of a head block
    int pk_grouped;            // packed: sequence by sequence in head blocks (else by pair level)
    int causal, packed;
    float scale_log2;          // scale * log2(e) (FP8: times the Q and K scales)
    float o_scale;             // FP8: the V scale, applied to O in the epilogue
    unsigned long long timeout_ns;
    unsigned long long* trace;     // FA_TRACE builds: per-role clock64 stamps of CTA 0
};

// Optional pipeline timeline (compile with -DFA_TRACE): CTA 0 records clock64
// stamps per role and iteration into Params::trace, laid out as
// [role][iteration][event], kTraceIters iterations and 8 events per role
// (roles 0, 1: the softmax warpgroups; 2, 3: the MMA issuer).
[[maybe_unused]] constexpr int kTraceIters = 1024;
#ifdef FA_TRACE
#define FA_TRACE_EV(role, it, ev)                                                              \
    do {                                                                                       \
        if (blockIdx.x == 0 && p.trace && (it) < kTraceIters)                                  \
            p.trace[((role) * kTraceIters + (it)) * 8 + (ev)] = clock64();                     \
    } while (0)
#else
#define FA_TRACE_EV(role, it, ev) \
    do {                          \
    } while (0)
#endif

struct Misc {
    uint64_t bar_q_full, bar_q_empty;
    uint64_t bar_kv_full[kMaxStages], bar_kv_empty[kMaxStages];
    uint64_t bar_s_full[2], bar_o_final[2], bar_drain;
    uint64_t bar_p_half[2][2];     // P_t keys 0-63 / 64-127 are in TMEM
    uint64_t bar_s_free[2];        // separate-P layout: the softmax warps have read S_t
    uint64_t bar_pv_done[2];       // separate-P layout: O_t += P_t V_j has completed
    uint64_t bar_feed_full[4], bar_feed_empty[4];   // the item ring (dynamic schedule)
    int feed[4];
    uint32_t tmem_base;
    int abort_flag;
    int bad;
    int total_items;
    int pmax;
};

// Packed batches only: the sequence offsets and the pair-level schedule.
struct SeqTables {
    int seq_off[kMaxSeqs + 1];
    int kseq_off[kMaxSeqs + 1];   // key offsets (equal to seq_off unless the queries are chunks)
    int order[kMaxSeqs];       // sequences by pair count, descending
    int pcnt[kMaxPairs];       // number of sequences with more than p pairs
    int pstart[kMaxPairs];     // first item index at pair level p
    // the dynamic schedule's order: sequence order[k]'s items start at item
    // sstart[k]; its heads run in blocks of gh[k] (K/V of a block fit the
    // L2 budget), each block's items heaviest pair first
    int sstart[kMaxSeqs];
    int gh[kMaxSeqs];
};

template <int D, bool PK, bool F8 = false>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kElem = F8 ? 1 : 2;                // bytes per element
    // bytes per tile row in shared memory: FP8 rows are always 128 bytes (at
    // d = 64 the TMA box's columns past d read as zeros, so the 128-byte
    // swizzled layout and the K = 128 score MMAs of d = 128 serve unchanged)
    static constexpr int kRowBytes = F8 ? 128 : D * kElem;
    static constexpr int kTileBytes = kBlockM * kRowBytes;  // one 128-row tile
    static constexpr int kBoxes = kRowBytes / 128;          // 128-byte-wide TMA boxes per tile row
    static constexpr int kBoxCols = 128 / kElem;            // elements per box row
    // K/V ring depth: what fits next to the two Q tiles (and the packed tables)
    static constexpr int kStages = F8 ? 10 : ((D == 128) ? (PK ? 4 : 5) : 10);
    static_assert(kStages <= kMaxStages, "ring");
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = 2 * kTileBytes;
    static constexpr int kMiscOff = kKVOff + kStages * kTileBytes;
    static constexpr int kTabOff = kMiscOff + (((int)sizeof(Misc) + 127) / 128) * 128;
    static constexpr int kSmemBytes = kTabOff + (PK ? (int)sizeof(SeqTables) : 0) + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory");
};

// One work item: two consecutive 128-row query tiles of one (sequence, head).
struct Item {
    int seq;       // batch index (dense) or sequence index (packed)
    int h;         // query head
    int q0;        // first row of tile 0 inside the sequence
    int len;       // query rows of the sequence
    int klen;      // keys of the sequence
    int qoff;      // position of query row 0 among the keys
    int tok0;      // packed: first token of the sequence
    int split;     // split of the key blocks this item covers (0 without splits)
    int j0;        // first key block of the item
    int n[2];      // key blocks each tile visits from j0 on (0: none)
};

// Position of query row `row` among the keys.
__device__ __forceinline__ int row_pos(int row, int qoff, int qmod) {
    return qoff + (qmod ? row % qmod : row);
}

// Key blocks a 128-row query tile starting at row q0 visits: all of them, or
// under the causal mask those up to the largest position of its valid rows.
__device__ __forceinline__ int tile_blocks(int q0, int len, int klen, int qoff, int qmod, int causal) {
    if (q0 >= len) return 0;
    const int nkv = (klen + kBlockN - 1) / kBlockN;
    if (!causal) return nkv;
    const int last = min(q0 + kBlockM - 1, len - 1);
    int last_pos;
    if (!qmod) {
        last_pos = qoff + last;
    } else {
        // rows q0 .. last cover positions q0 % qmod onwards, wrapping at qmod
        const int first = q0 % qmod;
        last_pos = qoff + ((last - q0 >= qmod - first) ? qmod - 1 : first + (last - q0));
    }
    return min(nkv, last_pos / kBlockN + 1);
}

// Dense batches: the (batch, head) units are cut into groups whose K/V fit in
// L2 together (query heads sharing a key/value head are adjacent); a group's
// items run in decreasing pair index (heaviest causal tiles first).  Packed
// batches: decreasing pair index over all sequences, then sequence, then head.
template <bool PK>
__device__ __forceinline__ Item decode_item(int idx, const Params& p, const Misc& ms, const SeqTables& tab) {
    Item it;
    int pair;
    if constexpr (!PK) {
        // units (b, h) in groups of group_units whose K/V fit in L2 together;
        // inside a group, heaviest pair first
        const int npairs = (p.N + kRowsPerItem - 1) / kRowsPerItem;
        it.split = idx % p.splits;              // the splits of one tile pair are adjacent items
        idx /= p.splits;
        const int per = p.B * p.Hq;
        const int G = p.group_units;
        const int g = idx / (npairs * G);
        const int gbase = g * G;
        const int gsz = min(G, per - gbase);
        const int r = idx - g * npairs * G;
        const int lvl = r / gsz;
        const int unit = gbase + (r - lvl * gsz);
        pair = npairs - 1 - lvl;
        it.seq = unit / p.Hq;
        it.h = unit - it.seq * p.Hq;
        it.len = p.N;
        it.klen = p.Nk;
        it.qoff = p.q_off;
        it.tok0 = 0;
    } else if (p.pk_grouped) {
        int lo = 0, hi = p.B - 1;          // last sorted sequence whose start <= idx
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tab.sstart[mid] <= idx) lo = mid; else hi = mid - 1;
        }
        it.seq = tab.order[lo];
        const int pk = (tab.seq_off[it.seq + 1] - tab.seq_off[it.seq] + kRowsPerItem - 1) / kRowsPerItem;
        const int gh = tab.gh[lo];
        const int r = idx - tab.sstart[lo];
        const int hb = min(r / (pk * gh), (p.Hq - 1) / gh);
        const int r2 = r - hb * pk * gh;
        const int bsz = min(gh, p.Hq - hb * gh);
        const int lvl = r2 / bsz;
        it.h = hb * gh + (r2 - lvl * bsz);
        pair = pk - 1 - lvl;
        it.tok0 = tab.seq_off[it.seq];
        it.len = tab.seq_off[it.seq + 1] - it.tok0;
        it.klen = tab.kseq_off[it.seq + 1] - tab.kseq_off[it.seq];
        it.qoff = p.causal ? it.klen - it.len : 0;     // a chunk's rows are the last positions
        it.split = 0;
    } else {
        int lo = 0, hi = ms.pmax - 1;      // smallest level whose start <= idx
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (tab.pstart[mid] <= idx) hi = mid; else lo = mid + 1;
        }
        pair = lo;
        const int rem = idx - tab.pstart[lo];
        const int k = rem / p.Hq;
        it.h = rem - k * p.Hq;
        it.seq = tab.order[k];
        it.tok0 = tab.seq_off[it.seq];
        it.len = tab.seq_off[it.seq + 1] - it.tok0;
        it.klen = tab.kseq_off[it.seq + 1] - tab.kseq_off[it.seq];
        it.qoff = p.causal ? it.klen - it.len : 0;     // a chunk's rows are the last positions
        it.split = 0;
    }
    it.q0 = pair * kRowsPerItem;
    const int qmod = PK ? 0 : p.qmod;
    it.n[0] = tile_blocks(it.q0, it.len, it.klen, it.qoff, qmod, p.causal);
    it.n[1] = tile_blocks(it.q0 + kBlockM, it.len, it.klen, it.qoff, qmod, p.causal);
    it.j0 = 0;
    if (!PK && p.splits > 1) {
        // split s covers key blocks [s * nmax / S, (s + 1) * nmax / S) of the
        // pair, nmax the larger block count of its two tiles
        const int nmax = max(it.n[0], it.n[1]);
        const int j0 = static_cast<int>(static_cast<long long>(it.split) * nmax / p.splits);
        const int j1 = static_cast<int>(static_cast<long long>(it.split + 1) * nmax / p.splits);
        it.j0 = j0;
        it.n[0] = max(0, min(j1, it.n[0]) - j0);
        it.n[1] = max(0, min(j1, it.n[1]) - j0);
    }
    return it;
}

// Static "snake" schedule over persistent CTAs: round r hands item
// r*G + c to CTA c on even rounds and r*G + (G-1-c) on odd rounds, which
// evens out the decreasing causal work between CTAs.
__device__ __forceinline__ int item_of_round(int r) {
    const int G = gridDim.x;
    return r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

// A waiting thread sleeps in try_wait (woken when the phase completes) instead
// of spinning, so it leaves issue slots to the softmax warps of its SM
// sub-partition; the sleep is bounded so that the timeout is still checked.
#ifndef FA_SUSPEND_NS
#define FA_SUSPEND_NS 20000u
#endif
constexpr uint32_t kSuspendNs = FA_SUSPEND_NS;

// Bounded wait: gives up after timeout_ns (recording the site in the status
// word and raising the CTA's abort flag) or as soon as another role aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Params& p, Misc& ms,
                                      int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
        if (*reinterpret_cast<volatile int*>(&ms.abort_flag)) return false;
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            *reinterpret_cast<volatile int*>(&ms.abort_flag) = 1;
            if (atomicCAS(p.status, 0, FA_ERR_DEVICE_TIMEOUT) == 0) {
                p.status[1] = site;
                p.status[2] = blockIdx.x;
            }
            return false;
        }
    }
}
// wait_bar on every lane of a warp, with one verdict for the whole warp
__device__ __forceinline__ bool wait_all(uint32_t bar, uint32_t parity, const Params& p, Misc& ms, int site) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, p, ms, site));
}
// Teardown wait: ignores the abort flag, still bounded.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, const Params& p) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > p.timeout_ns) return;
    }
}

// ------------------------------------------------------------ work feed
// Dynamic schedule (FA_DYN_SCHED, the default).  CTA c starts with item c;
// after that the producer thread takes the next item of the global order
// from a counter in global memory each time its CTA's loads of the previous
// item are all issued, and hands the index to the other roles through a ring
// of kFeedDepth slots in shared memory.  So every CTA takes the next item when
// it is about to be ready for one (a longest-first order then balances the
// CTAs), and the items in flight on the GPU at any time are consecutive in
// the order, i.e. come from the few (batch, head) units whose K/V share L2.
// The counter word carries the launch's epoch in its upper half.  A CTA that
// reads an earlier launch's epoch there swaps in {epoch, 0} with a
// compare-and-swap against the value it read; the word changes only through
// such a swap until it holds this launch's epoch (counting adds are made only
// after that has been seen), so exactly one swap succeeds and every failed one
// means the word has moved on.  So a launch needs no reset from the one
// before it, even an aborted one; a launch that ends normally also returns its
// word to {epoch, 0} (sched_take), for a replay with the same epoch (a CUDA
// graph).  Launches with few items per CTA (p.dyn = 0), and
// every launch of a build with FA_DYN_SCHED=0, follow the static snake of
// item_of_round instead.
#ifndef FA_DYN_SCHED
#define FA_DYN_SCHED 1
#endif
constexpr int kFeedDepth = 4;
// the next dynamic item (0, 1, ... in this launch); 0x3fffffff (no item,
// error recorded) if the word keeps changing under the swap, which only a
// launch of long ago still running on the same counter could cause.  Each
// CTA that takes at all stops after its first take past the last item, so a
// launch makes exactly `total` takes (`total` - G that succeed and one that
// fails per CTA, G = min(grid, total) CTAs); the take numbered total - 1 is
// the last and puts the word back to {epoch, 0}, so that a replay of the
// same launch (a CUDA graph, same epoch) starts from a clean count.
__device__ __forceinline__ int sched_take(const Params& p, Misc& ms, int total) {
    const unsigned long long tag = static_cast<unsigned long long>(p.epoch) << 32;
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(p.sched);
    for (int tries = 0; static_cast<unsigned>(cur >> 32) != p.epoch; ++tries) {
        if (tries == 64) {
            *reinterpret_cast<volatile int*>(&ms.abort_flag) = 1;
            if (atomicCAS(p.status, 0, FA_ERR_DEVICE_TIMEOUT) == 0) {
                p.status[1] = kSiteFeed;
                p.status[2] = blockIdx.x;
            }
            return 0x3fffffff;
        }
        const unsigned long long seen = atomicCAS(p.sched, cur, tag);
        // success: the word is now {epoch, 0}; failure: another CTA's swap
        // (the only other change an old-epoch word can see) moved it on
        cur = seen == cur ? tag : seen;
    }
    const int c = static_cast<int>(atomicAdd(p.sched, 1ull) & 0xffffffffull);
    if (c == total - 1) atomicExch(p.sched, tag);
    return c;
}
// item of round r for this CTA's producer (all items past the first are dynamic)
__device__ __forceinline__ int producer_item(const Params& p, Misc& ms, int r, int total) {
    if (!FA_DYN_SCHED || !p.dyn) return item_of_round(r);
    if (r == 0) return blockIdx.x;
    return min(static_cast<int>(gridDim.x) + sched_take(p, ms, total), total);
}
// a consumer warp takes its r-th item (all lanes; one arrival per warp)
__device__ __forceinline__ bool feed_take(const Params& p, Misc& ms, int r, int& idx) {
    if (!FA_DYN_SCHED || !p.dyn) {
        idx = item_of_round(r);
        return true;
    }
    if (r == 0) {
        idx = blockIdx.x;
        return true;
    }
    const uint32_t u = static_cast<uint32_t>(r - 1);     // rounds 1, 2, ... pass through the ring
    const uint32_t s = u % kFeedDepth;
    if (!wait_all(smem_u32(&ms.bar_feed_full[s]), (u / kFeedDepth) & 1u, p, ms, kSiteFeed)) return false;
    idx = *reinterpret_cast<volatile int*>(&ms.feed[s]);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&ms.bar_feed_empty[s]));
    return true;
}
// the producer thread publishes its r-th item (r >= 1; total: no more items)
__device__ __forceinline__ bool feed_give(const Params& p, Misc& ms, int r, int idx) {
    if (!FA_DYN_SCHED || !p.dyn) return true;
    if (r == 0) return true;
    const uint32_t u = static_cast<uint32_t>(r - 1);
    const uint32_t s = u % kFeedDepth;
    if (!wait_bar(smem_u32(&ms.bar_feed_empty[s]), ((u / kFeedDepth) & 1u) ^ 1u, p, ms, kSiteFeed)) return false;
    *reinterpret_cast<volatile int*>(&ms.feed[s]) = idx;
    mbar_arrive(smem_u32(&ms.bar_feed_full[s]));
    return true;
}

// ---------------------------------------------------------------- producer
template <int D, bool PK, bool F8 = false>
__device__ void load_role(const Params& p, Misc& ms, const SeqTables& tab, uint32_t smem_q, uint32_t smem_kv,
                          int total) {
    using C = Cfg<D, PK, F8>;
    const uint64_t pol_kv = policy_evict_last();
    const uint64_t pol_q = policy_evict_first();
    uint32_t kv_it = 0, item_n = 0;
    uint32_t st = 0, ph = 0;      // ring position of tile kv_it: stage and phase parity
    bool ok = true;
    for (int r = 0; ok; ++r) {
        // the next item, taken only now that this CTA's loads of its previous
        // item are all issued (taking it earlier would reserve it for a CTA
        // that may still be busy for long)
        const int idx = producer_item(p, ms, r, total);
        if (!(ok = feed_give(p, ms, r, idx))) break;
        if (idx >= total) break;
        const Item it = decode_item<PK>(idx, p, ms, tab);
        if (max(it.n[0], it.n[1]) == 0) continue;      // a split with no key block
        // both query tiles of the item
        if (!(ok = wait_bar(smem_u32(&ms.bar_q_empty), (item_n & 1) ^ 1, p, ms, kSiteQEmpty))) break;
        const uint32_t qbar = smem_u32(&ms.bar_q_full);
        mbar_arrive_expect_tx(qbar, 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t) {
            const int row = it.q0 + t * kBlockM;
            for (int b = 0; b < C::kBoxes; ++b) {
                const uint32_t dst = smem_q + t * C::kTileBytes + b * kBoxBytes;
                if constexpr (!PK)
                    tma_load_4d(dst, &p.tm_q, qbar, b * C::kBoxCols, row, it.h, it.seq, pol_q);
                else
                    tma_load_4d(dst, &p.tm_q, qbar, b * C::kBoxCols, it.h, it.tok0 + row, 0, pol_q);
            }
        }
        ++item_n;
        const int kvh = it.h / p.group;
        const int ktok0 = PK ? tab.kseq_off[it.seq] : 0;      // packed: the sequence's first key token
        const int nmax = max(it.n[0], it.n[1]);
        for (int j = 0; j < nmax && ok; ++j) {
            for (int kind = 0; kind < 2; ++kind) {       // K_j then V_j
                if (!(ok = wait_bar(smem_u32(&ms.bar_kv_empty[st]), ph ^ 1u, p, ms, kSiteKvEmpty))) break;
                const uint32_t bar = smem_u32(&ms.bar_kv_full[st]);
                mbar_arrive_expect_tx(bar, C::kTileBytes);
                const CUtensorMap* map = kind == 0 ? &p.tm_k : &p.tm_v;
                for (int b = 0; b < C::kBoxes; ++b) {
                    const uint32_t dst = smem_kv + st * C::kTileBytes + b * kBoxBytes;
                    const int key0 = (it.j0 + j) * kBlockN;
                    if constexpr (!PK)
                        tma_load_4d(dst, map, bar, b * C::kBoxCols, key0, kvh, it.seq, pol_kv);
                    else
                        tma_load_4d(dst, map, bar, b * C::kBoxCols, kvh, ktok0 + key0, 0, pol_kv);
                }
                ++kv_it;
                if (++st == (uint32_t)C::kStages) {
                    st = 0;
                    ph ^= 1u;
                }
            }
        }
    }
    if (!ok) {
        // let the copies already issued land before the CTA goes away
        if (item_n > 0) drain_bar(smem_u32(&ms.bar_q_full), (item_n - 1) & 1, p);
        const uint32_t first = kv_it > (uint32_t)C::kStages ? kv_it - C::kStages : 0;
        for (uint32_t i = first; i < kv_it; ++i)
            drain_bar(smem_u32(&ms.bar_kv_full[i % C::kStages]), (i / C::kStages) & 1, p);
    }
}

// ------------------------------------------------------------- MMA issuer
// S_t = Q_t K^T over K = d (steps of 16), both operands K-major, 128-byte
// swizzle; O_t (+)= P_t V with P read from TMEM.  Each is one asm block.
template <int D, bool F8 = false>
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint64_t dq, uint64_t dk) {
    if constexpr (F8) {
        umma_f8_ss_k128_x4(tmem_s, dq, dk, idesc_e4m3_f32(kBlockM, kBlockN, false));
    } else {
        constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, kBlockN, false);
        if constexpr (D == 128)
            umma_ss_k128_x8(tmem_s, dq, dk, idesc);
        else
            umma_ss_k64_x4(tmem_s, dq, dk, idesc);
    }
}
// Half h of O_t (+)= P_t V: keys 64h .. 64h+63 (bf16: P columns 32h.., FP8:
// P columns 16h..; V rows 64h.. of 128 bytes each)
template <int D, bool F8 = false>
__device__ __forceinline__ void issue_pv_half(uint32_t tmem_o, uint32_t tmem_p, uint64_t dv, int h, bool accumulate) {
    if constexpr (F8) {
        umma_f8_ts_kv64_x2(tmem_o, tmem_p + 16 * h, dv + static_cast<uint64_t>(h * ((64 * 128) >> 4)),
                           idesc_e4m3_f32(kBlockM, D, true), accumulate ? 1u : 0u);
    } else {
        constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, D, true);
        umma_ts_kv64_x4(tmem_o, tmem_p + 32 * h, dv + static_cast<uint64_t>(h * ((64 * 128) >> 4)), idesc,
                        accumulate ? 1u : 0u);
    }
}

// The MMA issuer.  Per work item it walks j = 0 .. nmax (nmax = the larger
// block count of the two tiles): O_t += P_t V_{j-1} for each tile that had
// block j-1, then S_t = Q_t K_j^T for each tile that has block j, tile 0
// before tile 1 -- the order that keeps the two softmax warpgroups out of phase.
// All 32 lanes of the warp run the loop (waits included); one elected lane
// issues each batch of MMAs and commits.
template <int D, bool PK, bool F8 = false>
__device__ void mma_role(const Params& p, Misc& ms, const SeqTables& tab, uint32_t tmem, uint32_t smem_q,
                         uint32_t smem_kv, int total) {
    using C = Cfg<D, PK, F8>;
    // descriptors of Q tile 0 and of ring stage 0; other tiles/stages are offsets
    const uint64_t dq0 = smem_desc_sw128(smem_q, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(smem_kv, 16, 1024);              // K-major (K tiles)
    const uint64_t dv0 = smem_desc_sw128(smem_kv, kBoxBytes, 1024);       // MN-major (V tiles)
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    // ring position (stage, phase parity) of the next K tile to consume; tiles
    // arrive in the order K_0, V_0, K_1, V_1, ... of each item
    uint32_t kst = 0, kph = 0, item_n = 0;
    uint32_t pc[2] = {0, 0};
    bool ok = true;
    for (int r = 0; ok; ++r) {
        int idx;
        if (!(ok = feed_take(p, ms, r, idx))) break;
        if (idx >= total) break;
        const Item it = decode_item<PK>(idx, p, ms, tab);
        if (max(it.n[0], it.n[1]) == 0) continue;      // a split with no key block
        if (!(ok = wait_all(smem_u32(&ms.bar_q_full), item_n & 1, p, ms, kSiteQFull))) break;
        tc_fence_after();
        ++item_n;
        const int nmax = max(it.n[0], it.n[1]);
        for (int j = 0; j <= nmax && ok; ++j) {
            FA_TRACE_EV(2, (item_n == 1 ? j : kTraceIters), 0);
            // V_{j-1} sits one ring position before K_j
            const uint32_t vst = kst == 0 ? C::kStages - 1 : kst - 1;
            const uint32_t vph = kst == 0 ? kph ^ 1u : kph;
            if (j > 0 && !(ok = wait_all(smem_u32(&ms.bar_kv_full[vst]), vph, p, ms, kSiteKvFull))) break;
            bool k_ready = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!ok) break;
                if (j > 0 && j - 1 < it.n[t]) {          // O_t += P_t V_{j-1}, in two key halves
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_p_half[t][h]), pc[t] & 1, p, ms, kSitePFull))) break;
                        tc_fence_after();
                        FA_TRACE_EV(3, (item_n == 1 ? j : kTraceIters), 2 * t + h);
                        if (h == 0) FA_TRACE_EV(2, (item_n == 1 ? j : kTraceIters), 2 + 2 * t);
                        if (elect_one())
                            issue_pv_half<D, F8>(tmem + 256 + t * 128, tmem + t * 128, dv0 + vst * kTileStep, h,
                                                 h > 0 || j - 1 > 0);
                        __syncwarp();
                    }
                    if (!ok) break;
                    ++pc[t];
                    if (j - 1 == it.n[t] - 1 && elect_one()) umma_commit(smem_u32(&ms.bar_o_final[t]));
                    __syncwarp();
                }
                if (j < it.n[t]) {                       // S_t = Q_t K_j^T
                    if (!k_ready) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_kv_full[kst]), kph, p, ms, kSiteKvFull))) break;
                        tc_fence_after();
                        k_ready = true;
                    }
                    if (elect_one()) {
                        issue_qk<D, F8>(tmem + t * 128, dq0 + t * kTileStep, dk0 + kst * kTileStep);
                        umma_commit(smem_u32(&ms.bar_s_full[t]));
                    }
                    __syncwarp();
                    FA_TRACE_EV(2, (item_n == 1 ? j : kTraceIters), 3 + 2 * t);
                }
            }
            if (!ok) break;
            if (elect_one()) {
                if (k_ready) umma_commit(smem_u32(&ms.bar_kv_empty[kst]));
                if (j > 0) umma_commit(smem_u32(&ms.bar_kv_empty[vst]));
                if (j == nmax - 1) umma_commit(smem_u32(&ms.bar_q_empty));
            }
            __syncwarp();
            if (j < nmax) {                               // next K tile: two positions on
                kst += 2;
                if (kst >= (uint32_t)C::kStages) {
                    kst -= C::kStages;
                    kph ^= 1u;
                }
            }
        }
    }
    // every MMA issued so far must be finished before TMEM and smem go away
    __syncwarp();
    if (elect_one()) umma_commit(smem_u32(&ms.bar_drain));
    __syncwarp();
    drain_bar(smem_u32(&ms.bar_drain), 0, p);
}

// The MMA issuer of the kSepP and kSharedS layouts (P in its own TMEM
// columns).  Per key block j it issues S_0(j), then S_1(j), each once the
// softmax warps have loaded the previous scores held in that S buffer
// (bar_s_free: per tile with kSepP, one for the shared buffer with kSharedS),
// and O_t += P_t(j-1) V_{j-1} for each tile once P_t(j-1) is written (two
// 64-key halves), each followed by a commit to bar_pv_done[t]: the softmax
// waits for it before it overwrites P_t or rescales O_t, and before its
// epilogue.  Order: kSepP  S_0(j) S_1(j) PV_0(j-1) PV_1(j-1);
//                   kSharedS S_0(j) PV_0(j-1) S_1(j) PV_1(j-1), so that a
// P V product runs while the shared scores are being read out.  K_j is
// released after the last S that reads it, V_{j-1} after the last P V, Q after
// the item's last S.
template <int D, bool PK, bool F8>
__device__ void mma_role_sep_p(const Params& p, Misc& ms, const SeqTables& tab, uint32_t tmem, uint32_t smem_q,
                               uint32_t smem_kv, int total) {
    using C = Cfg<D, PK, F8>;
    constexpr bool kShared = tmem_layout<D, F8>() == kSharedS;
    const uint64_t dq0 = smem_desc_sw128(smem_q, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(smem_kv, 16, 1024);              // K-major (K tiles)
    const uint64_t dv0 = smem_desc_sw128(smem_kv, kBoxBytes, 1024);       // MN-major (V tiles)
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    uint32_t kst = 0, kph = 0, item_n = 0;
    uint32_t pc[2] = {0, 0};      // P_t blocks consumed (phase parity of bar_p_half[t][*])
    uint32_t sn[2] = {0, 0};      // S issued into buffer 0 / 1: every S but the first waits for bar_s_free
    bool ok = true;
    for (int r = 0; ok; ++r) {
        int idx;
        if (!(ok = feed_take(p, ms, r, idx))) break;
        if (idx >= total) break;
        const Item it = decode_item<PK>(idx, p, ms, tab);
        if (max(it.n[0], it.n[1]) == 0) continue;      // a split with no key block
        if (!(ok = wait_all(smem_u32(&ms.bar_q_full), item_n & 1, p, ms, kSiteQFull))) break;
        tc_fence_after();
        ++item_n;
        const int nmax = max(it.n[0], it.n[1]);
        for (int j = 0; j <= nmax && ok; ++j) {
            // V_{j-1} sits one ring position before K_j
            const uint32_t vst = kst == 0 ? C::kStages - 1 : kst - 1;
            const uint32_t vph = kst == 0 ? kph ^ 1u : kph;
            bool k_ready = false, v_ready = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (j < it.n[t]) {                        // S_t = Q_t K_j^T
                    const int b = kShared ? 0 : t;        // S buffer
                    if (sn[b] > 0 &&
                        !(ok = wait_all(smem_u32(&ms.bar_s_free[b]), (sn[b] - 1) & 1, p, ms, kSiteSFree)))
                        break;
                    if (!k_ready) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_kv_full[kst]), kph, p, ms, kSiteKvFull))) break;
                        k_ready = true;
                    }
                    tc_fence_after();
                    if (elect_one()) {
                        issue_qk<D, F8>(tmem + tmem_s_col<D, F8>(t), dq0 + t * kTileStep, dk0 + kst * kTileStep);
                        umma_commit(smem_u32(&ms.bar_s_full[t]));
                        // the last S that reads K_j (and, at the item's end, Q)
                        if (t == 1 || j >= it.n[1]) {
                            umma_commit(smem_u32(&ms.bar_kv_empty[kst]));
                            if (j == nmax - 1) umma_commit(smem_u32(&ms.bar_q_empty));
                        }
                    }
                    __syncwarp();
                    ++sn[b];
                }
                // O_u += P_u V_{j-1}: tile u = t right after its S with the
                // shared buffer, both tiles after S_1 with separate buffers
#pragma unroll
                for (int u = kShared ? t : 0; u <= t; ++u) {
                    if (!kShared && t == 0) break;
                    if (j == 0 || j - 1 >= it.n[u]) continue;
                    if (!v_ready) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_kv_full[vst]), vph, p, ms, kSiteKvFull))) break;
                        v_ready = true;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_p_half[u][h]), pc[u] & 1, p, ms, kSitePFull))) break;
                        tc_fence_after();
                        if (elect_one())
                            issue_pv_half<D, F8>(tmem + tmem_o_col<D, F8>(u), tmem + tmem_p_col<D, F8>(u),
                                             dv0 + vst * kTileStep, h, h > 0 || j - 1 > 0);
                        __syncwarp();
                    }
                    if (!ok) break;
                    ++pc[u];
                    if (elect_one()) {
                        umma_commit(smem_u32(&ms.bar_pv_done[u]));
                        if (u == 1 || j - 1 >= it.n[1]) umma_commit(smem_u32(&ms.bar_kv_empty[vst]));
                    }
                    __syncwarp();
                }
                if (!ok) break;
            }
            if (!ok) break;
            if (j < nmax) {                               // next K tile: two positions on
                kst += 2;
                if (kst >= (uint32_t)C::kStages) {
                    kst -= C::kStages;
                    kph ^= 1u;
                }
            }
        }
    }
    // every MMA issued so far must be finished before TMEM and smem go away
    __syncwarp();
    if (elect_one()) umma_commit(smem_u32(&ms.bar_drain));
    __syncwarp();
    drain_bar(smem_u32(&ms.bar_drain), 0, p);
}

// Two issuers for the separate-P layouts: warp kMmaWarp issues the S
// products (each as soon as its S buffer is free), warp kAllocWarp the P V
// products (each as soon as its P is written), so that neither kind waits
// behind the other's barriers.  They walk the same items and ring positions:
// K_j at 2j, V_j at 2j + 1 from an item's first tile.
#ifndef FA_SPLIT_ISSUE
#define FA_SPLIT_ISSUE 1
#endif
template <int D, bool F8>
__host__ __device__ constexpr bool split_issue() {
    return sep_p<D, F8>() && FA_SPLIT_ISSUE;
}

#ifndef FA_PRE_DESC
#define FA_PRE_DESC 1
#endif
template <int D, bool PK, bool F8, bool PV>
__device__ void mma_role_split(const Params& p, Misc& ms, const SeqTables& tab, uint32_t tmem, uint32_t smem_q,
                               uint32_t smem_kv, int total) {
    using C = Cfg<D, PK, F8>;
    constexpr bool kShared = tmem_layout<D, F8>() == kSharedS;
    constexpr bool kPre = FA_PRE_DESC && !F8;
    // descriptor start-address steps of the 16-element K steps (128-byte
    // swizzle, K-major): +2 per step, +1024 for the second 64-column box;
    // V (MN-major): +128 per 16 key rows
    constexpr int kSteps = D / 16;
    const uint64_t dq0 = smem_desc_sw128(smem_q, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(smem_kv, 16, 1024);              // K-major (K tiles)
    const uint64_t dv0 = smem_desc_sw128(smem_kv, kBoxBytes, 1024);       // MN-major (V tiles)
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    uint32_t kst = 0, kph = 0, item_n = 0;    // ring position of the item's next K tile
    uint32_t pc[2] = {0, 0};      // P_t blocks consumed (phase parity of bar_p_half[t][*])
    uint32_t sn[2] = {0, 0};      // S issued into buffer 0 / 1: every S but the first waits for bar_s_free
    bool ok = true;
    for (int r = 0; ok; ++r) {
        int idx;
        if (!(ok = feed_take(p, ms, r, idx))) break;
        if (idx >= total) break;
        const Item it = decode_item<PK>(idx, p, ms, tab);
        if (max(it.n[0], it.n[1]) == 0) continue;      // a split with no key block
        if constexpr (!PV) {
            FA_TRACE_EV(2, kTraceIters - 32 + (item_n & 31), 6);
            if (!(ok = wait_all(smem_u32(&ms.bar_q_full), item_n & 1, p, ms, kSiteQFull))) break;
            tc_fence_after();
            FA_TRACE_EV(2, kTraceIters - 32 + (item_n & 31), 7);
        }
        ++item_n;
        const int nmax = max(it.n[0], it.n[1]);
        for (int j = 0; j < nmax && ok; ++j) {
            [[maybe_unused]] const int tj = item_n == 1 ? j : kTraceIters;     // timeline of the first item only
            FA_TRACE_EV(PV ? 3 : 2, tj, 0);
            if constexpr (!PV) {
                bool k_ready = false;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (j >= it.n[t]) continue;
                    const int b = kShared ? 0 : t;
                    if (sn[b] > 0 &&
                        !(ok = wait_all(smem_u32(&ms.bar_s_free[b]), (sn[b] - 1) & 1, p, ms, kSiteSFree)))
                        break;
                    if (!k_ready) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_kv_full[kst]), kph, p, ms, kSiteKvFull))) break;
                        k_ready = true;
                    }
                    tc_fence_after();
                    FA_TRACE_EV(2, tj, 1 + 2 * t);
                    if constexpr (kPre) {
                        uint64_t ad[kSteps], bd[kSteps];
#pragma unroll
                        for (int i = 0; i < kSteps; ++i) {
                            const uint64_t off = (i & 3) * 2 + (i >> 2) * 1024;
                            ad[i] = dq0 + t * kTileStep + off;
                            bd[i] = dk0 + kst * kTileStep + off;
                        }
                        if (elect_one()) {
                            constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, kBlockN, false);
                            FA_TRACE_EV(2, 512 + tj, 3 * t);
                            if constexpr (D == 128)
                                umma_ss_x8_pre(tmem + tmem_s_col<D, F8>(t), ad, bd, idesc);
                            else
                                umma_ss_x4_pre(tmem + tmem_s_col<D, F8>(t), ad, bd, idesc);
                            FA_TRACE_EV(2, 512 + tj, 3 * t + 1);
                            umma_commit(smem_u32(&ms.bar_s_full[t]));
                            if (t == 1 || j >= it.n[1]) {
                                umma_commit(smem_u32(&ms.bar_kv_empty[kst]));
                                if (j == nmax - 1) umma_commit(smem_u32(&ms.bar_q_empty));
                            }
                            FA_TRACE_EV(2, 512 + tj, 3 * t + 2);
                        }
                    } else if (elect_one()) {
                        issue_qk<D, F8>(tmem + tmem_s_col<D, F8>(t), dq0 + t * kTileStep, dk0 + kst * kTileStep);
                        umma_commit(smem_u32(&ms.bar_s_full[t]));
                        if (t == 1 || j >= it.n[1]) {
                            umma_commit(smem_u32(&ms.bar_kv_empty[kst]));
                            if (j == nmax - 1) umma_commit(smem_u32(&ms.bar_q_empty));
                        }
                    }
                    __syncwarp();
                    FA_TRACE_EV(2, tj, 2 + 2 * t);
                    ++sn[b];
                }
            } else {
                // V_j sits one ring position after K_j
                const uint32_t vst = kst + 1 == (uint32_t)C::kStages ? 0 : kst + 1;
                const uint32_t vph = kst + 1 == (uint32_t)C::kStages ? kph ^ 1u : kph;
                if (!(ok = wait_all(smem_u32(&ms.bar_kv_full[vst]), vph, p, ms, kSiteKvFull))) break;
                FA_TRACE_EV(3, tj, 1);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (j >= it.n[t]) continue;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(ok = wait_all(smem_u32(&ms.bar_p_half[t][h]), pc[t] & 1, p, ms, kSitePFull))) break;
                        tc_fence_after();
                        FA_TRACE_EV(3, tj, 2 + 3 * t + h);
                        if constexpr (kPre) {
                            uint32_t a[4];
                            uint64_t b[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                a[i] = tmem + tmem_p_col<D, F8>(t) + 32 * h + 8 * i;
                                b[i] = dv0 + vst * kTileStep + static_cast<uint64_t>(h * ((64 * 128) >> 4) + 128 * i);
                            }
                            if (elect_one())
                                umma_ts_x4_pre(tmem + tmem_o_col<D, F8>(t), a, b, idesc_bf16_f32(kBlockM, D, true),
                                               (h > 0 || j > 0) ? 1u : 0u);
                        } else if (elect_one()) {
                            issue_pv_half<D, F8>(tmem + tmem_o_col<D, F8>(t), tmem + tmem_p_col<D, F8>(t),
                                                 dv0 + vst * kTileStep, h, h > 0 || j > 0);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    ++pc[t];
                    if (elect_one()) {
                        umma_commit(smem_u32(&ms.bar_pv_done[t]));
                        if (t == 1 || j >= it.n[1]) umma_commit(smem_u32(&ms.bar_kv_empty[vst]));
                    }
                    __syncwarp();
                    FA_TRACE_EV(3, tj, 4 + 3 * t);
                }
            }
            if (!ok) break;
            kst += 2;                                     // next K tile: two positions on
            if (kst >= (uint32_t)C::kStages) {
                kst -= C::kStages;
                kph ^= 1u;
            }
        }
    }
    // every MMA this warp issued must be finished before TMEM and smem go
    // away (bar_drain takes one commit from each issuer)
    __syncwarp();
    if (elect_one()) umma_commit(smem_u32(&ms.bar_drain));
    __syncwarp();
    drain_bar(smem_u32(&ms.bar_drain), 0, p);
}

// ---------------------------------------------------------------- softmax
// exp2 of a pair of floats on the FMA pipe instead of the MUFU unit:
// 2^x = 2^j * 2^f with j = round(x), f = x - j in [-0.5, 0.5]; 2^f is a
// degree-3 minimax polynomial (max relative error 7.5e-5; coefficients fitted
// by fit_exp2_poly.py next to this file) and 2^j is added to the exponent
// field.  x is clamped at -126 so that the exponent never wraps; masked
// entries (-inf) then give 2^-126 instead of 0, which is below the fp32
// resolution of any row sum that holds the row maximum (>= 1).
#ifndef FA_POLY_PAIRS_PER8
#define FA_POLY_PAIRS_PER8 0
#endif
#ifndef FA_POLY_PAIRS_PER8_F8
#define FA_POLY_PAIRS_PER8_F8 1
#endif
// column pairs (of every 8) on the polynomial, per path: FP8 (tensor work per
// block half as long as bf16's, as many exponentials), bf16 d = 64 (the
// exponentials cost twice the block's MMAs), bf16 d = 128 (equal costs)
#ifndef FA_POLY_PAIRS_PER8_D64
#define FA_POLY_PAIRS_PER8_D64 2
#endif
template <int D, bool F8>
__host__ __device__ constexpr int poly_pairs_per8() {
    return F8 ? FA_POLY_PAIRS_PER8_F8 : (D == 64 ? FA_POLY_PAIRS_PER8_D64 : FA_POLY_PAIRS_PER8);
}
__device__ __forceinline__ uint64_t f2_const(uint32_t bits) {
    return (static_cast<uint64_t>(bits) << 32) | bits;
}
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
    float x0, x1;
    f2_unpack(x, x0, x1);
    x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t t = f2_add(x, f2_const(0x4B400000u));        // 1.5 * 2^23 + round(x)
    const uint64_t r = f2_add(t, f2_const(0xCB400000u));        // round(x)
    const uint64_t f = f2_fma(r, f2_const(0xBF800000u), x);     // x - round(x)
    uint64_t q = f2_fma(f2_const(0x3D61FBB0u), f, f2_const(0x3E786F0Du));   // c3 f + c2
    q = f2_fma(q, f, f2_const(0x3F31798Du));                                // .. f + c1
    q = f2_fma(q, f, f2_const(0x3F7FFB49u));                                // .. f + c0
    float q0, q1, t0, t1;
    f2_unpack(q, q0, q1);
    f2_unpack(t, t0, t1);
    q0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
    q1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
    return f2_pack(q0, q1);
}

// Row maximum of the 128 scores: four independent chains of 3-input max.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) {
    float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
    for (int c = 0; c < 128; c += 8) {
        m0 = fmax3(m0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        m1 = fmax3(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        m2 = fmax3(m2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
        m3 = fmax3(m3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
    }
    return fmax3(fmaxf(m0, m1), m2, m3);
}

// Exponentials of key half HALF (columns 64*HALF .. +63) of a score row:
// p = 2^(s * scale_log2 - msub) with nm2 = (-msub, -msub), packed into pk
// (bf16 pairs; FP8: four E4M3 per word in pk[0..15]), their fp32 sums added
// pairwise into acc.  NPOLY column pairs of every 8 take the FMA-pipe
// polynomial, the rest ex2 on MUFU.
template <bool F8, int HALF, int NPOLY>
__device__ __forceinline__ void exp_half(const uint32_t (&s)[128], uint64_t sl2x2, uint64_t nm2, uint32_t (&pk)[32],
                                         uint64_t (&acc)[4]) {
    float e_prev = 0.f, e_prev1 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int gi = 32 * HALF + i;       // pair of columns 2gi, 2gi+1
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[2 * gi]), __uint_as_float(s[2 * gi + 1])), sl2x2, nm2);
        uint64_t e;
        if ((gi % 8) < NPOLY) {
            e = exp2_poly2(x);
        } else {
            float x0, x1;
            f2_unpack(x, x0, x1);
            e = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        acc[i & 3] = f2_add(acc[i & 3], e);
        float e0, e1;
        f2_unpack(e, e0, e1);
        if constexpr (F8) {
            // P <= 2^8 fits E4M3's range (448)
            if (i & 1)
                pk[i >> 1] = pack_e4m3x4(e_prev, e_prev1, e0, e1);
            else {
                e_prev = e0;
                e_prev1 = e1;
            }
        } else {
            pk[i] = pack_bf16x2(e0, e1);
        }
    }
}

template <int D, bool PK, bool F8 = false>
__device__ void softmax_role(const Params& p, Misc& ms, const SeqTables& tab, uint32_t tmem, int warp, int lane,
                             int total) {
    const int t = warp / 4;                          // query tile of this warpgroup
    const int wq = warp % 4;                         // TMEM lane quarter
    const int r = wq * 32 + lane;                    // row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    constexpr bool SP = sep_p<D, F8>();
    const uint32_t taddr_s = tmem + lane_off + tmem_s_col<D, F8>(t);
    const uint32_t taddr_p = tmem + lane_off + tmem_p_col<D, F8>(t);
    const int sfree = tmem_layout<D, F8>() == kSharedS ? 0 : t;     // barrier of this tile's S buffer
    const uint32_t taddr_o = tmem + lane_off + tmem_o_col<D, F8>(t);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    uint32_t sc = 0, oc = 0, pw = 0;     // S blocks, O finals, P V completions waited for

    bool ok = true;
    for (int rr = 0; ok; ++rr) {
        // (feed_take's cases spelled out: this form keeps the loop free of spills)
        int idx = item_of_round(rr);
        if (FA_DYN_SCHED && p.dyn && rr > 0) {
            if (!feed_take(p, ms, rr, idx)) {
                ok = false;
                break;
            }
        } else if (FA_DYN_SCHED && p.dyn) {
            idx = blockIdx.x;
        }
        if (idx >= total) break;
        const Item it = decode_item<PK>(idx, p, ms, tab);
        const int n = t ? it.n[1] : it.n[0];
        const int row = it.q0 + t * kBlockM + r;
        if (n == 0) {
            // a split that holds no key block of this tile contributes nothing
            if (!PK && p.o_part != nullptr && row < it.len)
                p.lse_part[static_cast<size_t>(it.split) * p.B * p.Hq * p.N +
                           (static_cast<size_t>(it.seq) * p.Hq + it.h) * p.N + row] = -INFINITY;
            continue;
        }
        // keys [0, limit) are allowed for this row (causal: up to its own position)
        const int limit = p.causal ? min(row_pos(row, it.qoff, PK ? 0 : p.qmod) + 1, it.klen) : it.klen;
        float m_used = -INFINITY;    // max the exponentials are taken against (log2 units)
        float l = 0.f;               // running sum of exp2(x - m_used)
        for (int j = 0; j < n; ++j) {
            if (lane == 0 && wq == 0) FA_TRACE_EV(t, sc, 0);
            ok = wait_bar(smem_u32(&ms.bar_s_full[t]), sc & 1, p, ms, kSiteSFull);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ++sc;
            tc_fence_after();
            if (lane == 0 && wq == 0) FA_TRACE_EV(t, sc - 1, 1);
            uint32_t s[128];
            tmem_ld128_sync(taddr_s, s);
            if constexpr (SP) {
                // the scores are in registers: S_t may take the next block
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ms.bar_s_free[sfree]));
            }
            if (lane == 0 && wq == 0) FA_TRACE_EV(t, sc - 1, 2);
            // separate P: P_t and O_t may be written once P_t V_{j-1} is done
            bool pv_free = !SP || j == 0;
            if ((it.j0 + j) * kBlockN + kBlockN > limit) {      // diagonal or tail block
                const int lim = limit - (it.j0 + j) * kBlockN;
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= lim) s[c] = __float_as_uint(-INFINITY);
            }
            constexpr int kPoly = poly_pairs_per8<D, F8>();
            // bf16: lazy rescale (the reference may trail the true maximum by
            // up to 2^8); FP8: threshold kF8Threshold with P computed as
            // 2^kF8Shift * exp2(x - m) <= 2^8.75 < 448, so that E4M3 holds every
            // entry above 2^-(6 + kF8Shift) of the row maximum as a normal number
            // (relative rounding error <= 2^-4); l carries the same factor, and
            // lse takes it back out
            constexpr float kThr = F8 ? kF8Threshold : kRescaleThreshold;
            constexpr float kPShift = F8 ? kF8Shift : 0.f;
            uint64_t acc[4] = {0, 0, 0, 0};      // packed row sums (+0.0f pairs)
            uint32_t pk[32];
            const float mx = row_max128(s);
            const float m_new = fmaxf(m_used, mx * sl2);
            if (lane == 0 && wq == 0) FA_TRACE_EV(t, sc - 1, 3);
            const bool need = m_new > m_used + kThr;
            const bool any_need = __any_sync(0xffffffffu, need);
            if (j > 0 && any_need) {
                // Theorem 2: rescale the partial output when the max grows.
                // Shared S/P: S_t(j) was issued after O_t += P_t V_{j-1}, so O_t
                // is final here; separate P: wait for that product first.
                if (!pv_free) {
                    ok = wait_bar(smem_u32(&ms.bar_pv_done[t]), pw & 1, p, ms, kSitePvDone);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    ++pw;
                    pv_free = true;
                    tc_fence_after();
                }
                const float f = need ? ex2_approx(m_used - m_new) : 1.f;
                const uint64_t f2 = f2_pack(f, f);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32_sync(taddr_o + c * 32, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float a, b;
                        f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), f2), a, b);
                        o[2 * i] = __float_as_uint(a);
                        o[2 * i + 1] = __float_as_uint(b);
                    }
                    tmem_st32(taddr_o + c * 32, o);
                }
                tmem_wait_st();
            }
            if (need) {
                l *= (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
                m_used = m_new;
            }
            const float msub = ((m_used == -INFINITY) ? 0.f : m_used) - kPShift;
            const uint64_t nm2 = f2_pack(-msub, -msub);
            exp_half<F8, 0, kPoly>(s, sl2x2, nm2, pk, acc);
            if (!pv_free) {
                ok = wait_bar(smem_u32(&ms.bar_pv_done[t]), pw & 1, p, ms, kSitePvDone);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ++pw;
                pv_free = true;
                tc_fence_after();
            }
            if constexpr (F8)
                tmem_st16(taddr_p, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
            else
                tmem_st32(taddr_p, pk);
            // keys 0-63 of P are ready: the tensor core can start on them
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ms.bar_p_half[t][0]));
            uint32_t pk1[32];
            exp_half<F8, 1, kPoly>(s, sl2x2, nm2, pk1, acc);
            if constexpr (F8)
                tmem_st16(taddr_p + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk1[0]));
            else
                tmem_st32(taddr_p + 32, pk1);
            {
                float a, b;
                f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a, b);
                l += a + b;
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) FA_TRACE_EV(t, sc - 1, wq == 0 ? 4 : 4 + wq);
            if (lane == 0) mbar_arrive(smem_u32(&ms.bar_p_half[t][1]));

        }
        if (!ok) break;
        // epilogue: O / l -> bf16 -> HBM, and the logsumexp
        if constexpr (SP) {
            ok = wait_bar(smem_u32(&ms.bar_pv_done[t]), pw & 1, p, ms, kSitePvDone);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ++pw;
        } else {
            ok = wait_bar(smem_u32(&ms.bar_o_final[t]), oc & 1, p, ms, kSiteOFinal);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ++oc;
        }
        tc_fence_after();
        const bool valid = row < it.len;
        float inv = l > 0.f ? 1.f / l : 0.f;
        if constexpr (F8) inv *= p.o_scale;
        uint16_t* orow;
        float* lrow;
        if constexpr (!PK) {
            const size_t rid = (static_cast<size_t>(it.seq) * p.Hq + it.h) * p.N + row;
            if (p.o_part != nullptr) {
                // this split's O / l in fp32 and its logsumexp; a combine pass
                // merges the splits
                const size_t prid = static_cast<size_t>(it.split) * p.B * p.Hq * p.N + rid;
                float* prow = p.o_part + prid * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32_sync(taddr_o + c * 32, o);
                    if (valid) {
                        float4* dst = reinterpret_cast<float4*>(prow + c * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                                 __uint_as_float(o[4 * i + 2]) * inv,
                                                 __uint_as_float(o[4 * i + 3]) * inv);
                    }
                }
                if (valid) {
                    float lg;
                    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    p.lse_part[prid] = (l > 0.f) ? (m_used + lg - (F8 ? kF8Shift : 0.f)) * 0.69314718055994531f : -INFINITY;
                }
                tc_fence_before();
                continue;
            }
            orow = static_cast<uint16_t*>(p.o) + rid * D;
            lrow = p.lse + rid;
        } else {
            const size_t tok = static_cast<size_t>(it.tok0) + row;
            orow = static_cast<uint16_t*>(p.o) + (tok * p.Hq + it.h) * D;
            lrow = p.lse + static_cast<size_t>(it.h) * p.N + tok;
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32_sync(taddr_o + c * 32, o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
        if (valid) {
            float lg;
            asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(lg) : "f"(l));
            *lrow = (l > 0.f) ? (m_used + lg - (F8 ? kF8Shift : 0.f)) * 0.69314718055994531f : -INFINITY;
        }
        tc_fence_before();
    }
}

// ------------------------------------------------------------------ kernel
template <int D, bool PK, bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_kernel(const __grid_constant__ Params p) {
    using C = Cfg<D, PK, F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc& ms = *reinterpret_cast<Misc*>(smem + C::kMiscOff);
    SeqTables& tab = *reinterpret_cast<SeqTables*>(smem + C::kTabOff);   // packed batches only
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const uint32_t smem_q = smem_u32(smem + C::kQOff);
    const uint32_t smem_kv = smem_u32(smem + C::kKVOff);

    if (tid == 0) {
        mbar_init(smem_u32(&ms.bar_q_full), 1);
        mbar_init(smem_u32(&ms.bar_q_empty), 1);
        mbar_init(smem_u32(&ms.bar_drain), split_issue<D, F8>() ? 2 : 1);
        for (int s = 0; s < kFeedDepth; ++s) {
            mbar_init(smem_u32(&ms.bar_feed_full[s]), 1);
            // consumers: the softmax warps and the MMA issuer warp(s)
            mbar_init(smem_u32(&ms.bar_feed_empty[s]), kNumSoftmaxWarps + (split_issue<D, F8>() ? 2 : 1));
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&ms.bar_kv_full[s]), 1);
            mbar_init(smem_u32(&ms.bar_kv_empty[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&ms.bar_s_full[t]), 1);
            mbar_init(smem_u32(&ms.bar_p_half[t][0]), 4); // one arrival per warp
            mbar_init(smem_u32(&ms.bar_p_half[t][1]), 4);
            mbar_init(smem_u32(&ms.bar_o_final[t]), 1);
            mbar_init(smem_u32(&ms.bar_s_free[t]), 4);     // one arrival per warp
            mbar_init(smem_u32(&ms.bar_pv_done[t]), 1);
        }
        ms.abort_flag = 0;
        ms.bad = 0;
        fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tensormap(&p.tm_q);
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
    }

    int total;
    if constexpr (PK) {
        // stage the offsets, check them, and build the pair-level tables
        for (int i = tid; i <= p.B; i += kThreads) {
            tab.seq_off[i] = p.cu_seqlens[i];
            tab.kseq_off[i] = p.cu_seqlens_k ? p.cu_seqlens_k[i] : p.cu_seqlens[i];
        }
        __syncthreads();
        if (tid == 0) {
            int bad = tab.seq_off[0] != 0 || tab.seq_off[p.B] != p.N || tab.kseq_off[0] != 0 ||
                      tab.kseq_off[p.B] != p.Nk;
            for (int s = 0; s < p.B && !bad; ++s) {
                const int L = tab.seq_off[s + 1] - tab.seq_off[s];
                const int Lk = tab.kseq_off[s + 1] - tab.kseq_off[s];
                if (L < 0 || L > kMaxPairs * kRowsPerItem || Lk < 0) bad = 1;
                if (p.causal && Lk < L) bad = 1;       // a chunk's rows are the last Lk positions
                if (!p.causal && L > 0 && Lk == 0) bad = 1;
            }
            ms.bad = bad;
        }
        __syncthreads();
        if (ms.bad) {
            if (tid == 0 && blockIdx.x == 0) atomicCAS(p.status, 0, FA_ERR_SEQLENS);
            return;
        }
        for (int s = tid; s < p.B; s += kThreads) {
            const int ps = (tab.seq_off[s + 1] - tab.seq_off[s] + kRowsPerItem - 1) / kRowsPerItem;
            int rank = 0;
            for (int u = 0; u < p.B; ++u) {
                const int pu = (tab.seq_off[u + 1] - tab.seq_off[u] + kRowsPerItem - 1) / kRowsPerItem;
                rank += (pu > ps) || (pu == ps && u < s);
            }
            tab.order[rank] = s;
        }
        __syncthreads();
        if (tid == 0) {
            auto pairs_of = [&](int s) {
                return (tab.seq_off[s + 1] - tab.seq_off[s] + kRowsPerItem - 1) / kRowsPerItem;
            };
            const int pmax = p.B > 0 ? pairs_of(tab.order[0]) : 0;
            int k = p.B;
            for (int lvl = 0; lvl < pmax; ++lvl) {
                while (k > 0 && pairs_of(tab.order[k - 1]) <= lvl) --k;
                tab.pcnt[lvl] = k;
            }
            int acc = 0;
            for (int lvl = pmax - 1; lvl >= 0; --lvl) {
                tab.pstart[lvl] = acc;
                acc += tab.pcnt[lvl] * p.Hq;
            }
            ms.pmax = pmax;
            ms.total_items = acc;
            int acc2 = 0;
            for (int k = 0; k < p.B; ++k) {
                const int sq = tab.order[k];
                const long long kv = 2ll * C::kElem * D * max(1, tab.kseq_off[sq + 1] - tab.kseq_off[sq]);
                const long long g = max(1ll, p.l2_group_bytes / kv) * p.group;   // whole GQA groups
                tab.gh[k] = static_cast<int>(min(g, static_cast<long long>(p.Hq)));
                tab.sstart[k] = acc2;
                acc2 += pairs_of(sq) * p.Hq;
            }
        }
    }

    if (warp == kAllocWarp) {
        tmem_alloc(smem_u32(&ms.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    if constexpr (PK) {
        total = ms.total_items;
    } else {
        total = ((p.N + kRowsPerItem - 1) / kRowsPerItem) * p.B * p.Hq * p.splits;
    }

    if (warp < kNumSoftmaxWarps) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        softmax_role<D, PK, F8>(p, ms, tab, tmem, warp, lane, total);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
        if (split_issue<D, F8>() && (warp == kMmaWarp || warp == kAllocWarp)) {
            if (warp == kMmaWarp)
                mma_role_split<D, PK, F8, false>(p, ms, tab, tmem, smem_q, smem_kv, total);
            else
                mma_role_split<D, PK, F8, true>(p, ms, tab, tmem, smem_q, smem_kv, total);
            __syncwarp();
        } else if (warp == kMmaWarp) {
            if constexpr (sep_p<D, F8>())
                mma_role_sep_p<D, PK, F8>(p, ms, tab, tmem, smem_q, smem_kv, total);   // all 32 lanes
            else
                mma_role<D, PK, F8>(p, ms, tab, tmem, smem_q, smem_kv, total);   // all 32 lanes
            __syncwarp();
        } else if (warp == kLoadWarp) {
            if (lane == 0) load_role<D, PK, F8>(p, ms, tab, smem_q, smem_kv, total);
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kAllocWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of the key splits (Theorem 2 applied to whole splits): with split s
// holding O_s = (its P V) / l_s and lse_s = m_s + ln l_s, the row's result is
// lse = ln sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) O_s.  One warp per
// row; each lane owns D / 32 consecutive columns.  Splits with no allowed key
// (lse_s = -inf) carry weight 0 and their O_s is not read; a row with no
// allowed key at all gets O = 0 and lse = -inf.
template <int D>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part, uint16_t* o, float* lse,
                                                         long long rows, int splits) {
    constexpr int kCols = D / 32;
    const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, lse_part[s * rows + row]);
    float acc[kCols];
#pragma unroll
    for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    if (mx != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = lse_part[s * rows + row];
            if (ls == -INFINITY) continue;
            const float w = __expf(ls - mx);
            wsum += w;
            const float* src = o_part + (static_cast<size_t>(s) * rows + row) * D + lane * kCols;
            if constexpr (kCols == 4) {
                const float4 v = *reinterpret_cast<const float4*>(src);
                acc[0] += w * v.x;
                acc[1] += w * v.y;
                acc[2] += w * v.z;
                acc[3] += w * v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(src);
                acc[0] += w * v.x;
                acc[1] += w * v.y;
            }
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint32_t pk[kCols / 2];
#pragma unroll
    for (int i = 0; i < kCols / 2; ++i) pk[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    uint16_t* dst = o + row * D + lane * kCols;
    if constexpr (kCols == 4)
        *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
    else
        *reinterpret_cast<uint32_t*>(dst) = pk[0];
    if (lane == 0) lse[row] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

// Watchdog self-test: one thread waits, through the same bounded wait the
// kernel's roles use, on an mbarrier that nothing ever arrives at.  The wait
// gives up after p.timeout_ns and records FA_ERR_DEVICE_TIMEOUT in the status
// word; the kernel then returns normally.
__global__ void fa_watchdog_probe_kernel(const __grid_constant__ Params p) {
    __shared__ Misc ms;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&ms.bar_q_full), 1);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)wait_bar(smem_u32(&ms.bar_q_full), 0, p, ms, kSiteQFull);
}

// =================================================================== host
static DeviceState g_dev[kMaxDevices];
static std::mutex g_mu;
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int init_device(int dev, DeviceState** out) {
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& ds = g_dev[dev];
    if (!ds.init) {
        ds.init = true;
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            ds.status_code = FA_ERR_LAUNCH;
        } else if (prop.major != 10 || prop.minor != 0) {
            ds.status_code = FA_ERR_ARCH;
        } else {
            ds.num_sms = prop.multiProcessorCount;
            if (!g_encode) {
                cudaDriverEntryPointQueryResult q;
                void* fn = nullptr;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                        cudaSuccess &&
                    q == cudaDriverEntryPointSuccess)
                    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
            bool good = g_encode != nullptr;
            good = good && cudaMalloc(&ds.status, 4 * sizeof(int)) == cudaSuccess;
            good = good && cudaMemset(ds.status, 0, 4 * sizeof(int)) == cudaSuccess;
            good = good && cudaMalloc(&ds.sched, kSchedSlots * sizeof(unsigned long long)) == cudaSuccess;
            good = good && cudaMemset(ds.sched, 0, kSchedSlots * sizeof(unsigned long long)) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, false>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, false>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, false, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, false, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, true, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, true, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, false, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, false, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, true, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, true, true>::kSmemBytes) == cudaSuccess;
            ds.status_code = good ? FA_OK : FA_ERR_LAUNCH;
        }
    }
    *out = &ds;
    return ds.status_code;
}

// 4-D bf16 tensor map with a 64 x rows box, 128-byte swizzle.
bool encode_map(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                const uint32_t box[4], bool bytes) {
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                          const_cast<void*>(base), dims, strides, box,
                          elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static bool make_maps(Params& P, const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int N,
                      int Nk, int d, bool packed, bool fp8 = false) {
    const uint64_t e = fp8 ? 1 : 2;
    if (!packed) {
        const uint64_t dq[4] = {(uint64_t)d, (uint64_t)N, (uint64_t)Hq, (uint64_t)B};
        const uint64_t sq[3] = {d * e, (uint64_t)N * d * e, (uint64_t)Hq * N * d * e};
        const uint64_t dk[4] = {(uint64_t)d, (uint64_t)Nk, (uint64_t)Hkv, (uint64_t)B};
        const uint64_t sk[3] = {d * e, (uint64_t)Nk * d * e, (uint64_t)Hkv * Nk * d * e};
        const uint32_t box[4] = {(uint32_t)(128 / e), (uint32_t)kBlockM, 1, 1};    // 128-byte box rows
        return encode_map(&P.tm_q, q, dq, sq, box, fp8) && encode_map(&P.tm_k, k, dk, sk, box, fp8) &&
               encode_map(&P.tm_v, v, dk, sk, box, fp8);
    }
    const uint64_t dq[4] = {(uint64_t)d, (uint64_t)Hq, (uint64_t)N, 1};
    const uint64_t sq[3] = {d * e, (uint64_t)Hq * d * e, (uint64_t)N * Hq * d * e};
    const uint64_t dk[4] = {(uint64_t)d, (uint64_t)Hkv, (uint64_t)Nk, 1};
    const uint64_t sk[3] = {d * e, (uint64_t)Hkv * d * e, (uint64_t)Nk * Hkv * d * e};
    const uint32_t box[4] = {(uint32_t)(128 / e), 1, (uint32_t)kBlockM, 1};      // 128-byte box rows
    return encode_map(&P.tm_q, q, dq, sq, box, fp8) && encode_map(&P.tm_k, k, dk, sk, box, fp8) &&
           encode_map(&P.tm_v, v, dk, sk, box, fp8);
}

// The dynamic schedule runs the items of groups of (batch, head) units whose
// K/V fit in this many MiB of L2 (126 MB) one group after the other.
#ifndef FA_L2_GROUP_MIB
#define FA_L2_GROUP_MIB 32ll
#endif
// Launches with fewer items than this many per SM keep the static snake
// (a CTA's one or two items: nothing to balance, and no counter to wait on).
#ifndef FA_DYN_MIN_ITEMS_PER_SM
#define FA_DYN_MIN_ITEMS_PER_SM 4
#endif

#ifdef FA_TRACE
static unsigned long long* g_trace = nullptr;
#endif

static bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

// the work counter and epoch of this device's next forward launch: launch n
// takes counter n % kSchedSlots with epoch n / kSchedSlots + 1
struct Sched {
    unsigned long long* word;
    unsigned epoch;
};
static Sched next_sched(std::atomic<unsigned>& seq, unsigned long long* words, unsigned slots) {
    const unsigned n = seq.fetch_add(1, std::memory_order_relaxed);
    return Sched{words + n % slots, n / slots + 1u};
}
static Sched next_sched(DeviceState* ds) { return next_sched(ds->sched_seq, ds->sched, kSchedSlots); }


// Fills the launch parameters and launches the kernel variant for (d, packed)
// on `stream`.  Nk / q_off describe a dense query chunk (Nk keys per sequence,
// query row 0 at key position q_off); a plain forward has Nk = N, q_off = 0.
// qmod, splits, o_part, lse_part: see Params (a plain forward has 0, 1, NULL, NULL).
static int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                      int N, int Nk, int q_off, int d, float scale, int causal, const int32_t* cu_seqlens,
                      cudaStream_t s, int* status, int num_sms, Sched sched, int qmod = 0, int splits = 1,
                      float* o_part = nullptr, float* lse_part = nullptr, bool fp8 = false,
                      float qk_scale = 1.f, float v_scale = 1.f, const int32_t* cu_seqlens_k = nullptr) {
    const bool packed = cu_seqlens != nullptr;
    Params P;
    std::memset(&P, 0, sizeof(P));
    if (!make_maps(P, q, k, v, B, Hq, Hkv, N, Nk, d, packed, fp8)) return FA_ERR_LAUNCH;
    P.o = o;
    P.lse = lse;
    P.cu_seqlens = cu_seqlens;
    P.cu_seqlens_k = cu_seqlens_k;
    P.status = status;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.N = N;
    P.Nk = Nk;
    P.q_off = q_off;
    P.group = Hq / Hkv;
    // work items: dense, known here; packed, counted on the device (at least
    // one per sequence and head per 256 tokens)
    const long long items = packed ? std::max<long long>(1, (long long)N / kRowsPerItem) * Hq
                                   : (long long)((N + kRowsPerItem - 1) / kRowsPerItem) * B * Hq * splits;
    P.dyn = (FA_DYN_SCHED && items >= (long long)FA_DYN_MIN_ITEMS_PER_SM * num_sms) ? 1 : 0;
    P.sched = sched.word;
    P.epoch = sched.epoch;
    {
        // dynamic schedule: K/V of one group of units stay resident in L2
        // while the group's items run; static: one group
        const long long kv_bytes = 4ll * Nk * d;                   // K and V of one kv head
        long long g_kv = std::max(1ll, (FA_L2_GROUP_MIB << 20) / std::max(1ll, kv_bytes));
        long long G = P.dyn ? std::min<long long>(g_kv * P.group, (long long)B * Hq) : (long long)B * Hq;
        P.group_units = (int)std::max(1ll, G);
        P.l2_group_bytes = FA_L2_GROUP_MIB << 20;
        // packed batches in the dynamic schedule: sequence by sequence (longest
        // first) in blocks of heads whose K/V fit the budget.  Not for FP8,
        // whose half-size K/V already hit L2 more often and whose packed
        // batch measured faster in the pair-level order
        P.pk_grouped = (packed && P.dyn && !fp8) ? 1 : 0;
    }
    P.causal = causal ? 1 : 0;
    P.packed = packed ? 1 : 0;
    P.scale_log2 = scale * qk_scale * 1.4426950408889634f;
    P.o_scale = v_scale;
    P.timeout_ns = 2000000000ull;
    P.qmod = qmod;
    P.splits = splits;
    P.o_part = o_part;
    P.lse_part = lse_part;
#ifdef FA_TRACE
    P.trace = g_trace;
#endif
    // dense: one CTA per item up to one per SM; packed: one per SM (the CTAs
    // with no item of the device's count return at once)
    const int grid = packed ? num_sms : (int)std::min<long long>(items, num_sms);
    if (fp8 && d == 64 && packed)
        fa_fwd_kernel<64, true, true><<<grid, kThreads, Cfg<64, true, true>::kSmemBytes, s>>>(P);
    else if (fp8 && d == 64)
        fa_fwd_kernel<64, false, true><<<grid, kThreads, Cfg<64, false, true>::kSmemBytes, s>>>(P);
    else if (fp8 && packed)
        fa_fwd_kernel<128, true, true><<<grid, kThreads, Cfg<128, true, true>::kSmemBytes, s>>>(P);
    else if (fp8)
        fa_fwd_kernel<128, false, true><<<grid, kThreads, Cfg<128, false, true>::kSmemBytes, s>>>(P);
    else if (d == 64 && !packed)
        fa_fwd_kernel<64, false><<<grid, kThreads, Cfg<64, false>::kSmemBytes, s>>>(P);
    else if (d == 64)
        fa_fwd_kernel<64, true><<<grid, kThreads, Cfg<64, true>::kSmemBytes, s>>>(P);
    else if (!packed)
        fa_fwd_kernel<128, false><<<grid, kThreads, Cfg<128, false>::kSmemBytes, s>>>(P);
    else
        fa_fwd_kernel<128, true><<<grid, kThreads, Cfg<128, true>::kSmemBytes, s>>>(P);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace fa_sm100

using namespace fa_sm100;

#ifdef FA_TRACE
extern "C" int fa_trace_set_buffer(void* dev_ptr) {
    fa_sm100::g_trace = static_cast<unsigned long long*>(dev_ptr);
    return FA_OK;
}
#endif

extern "C" int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                      int N, int d, float scale, int causal, const int32_t* cu_seqlens, void* stream) {
    const bool packed = cu_seqlens != nullptr;
    if (B < 0 || N < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if (packed && (B > kMaxSeqs || !aligned(cu_seqlens, 4))) return B > kMaxSeqs ? FA_ERR_SHAPE : FA_ERR_ALIGN;
    // row ids and item counts must fit in int
    const long long rows = packed ? (long long)Hq * N : (long long)B * Hq * N;
    if (rows > (1ll << 30)) return FA_ERR_SHAPE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;

    return launch_fwd(q, k, v, o, lse, B, Hq, Hkv, N, N, 0, d, scale, causal, cu_seqlens,
                      static_cast<cudaStream_t>(stream), ds->status, ds->num_sms, next_sched(ds));
}

extern "C" int fa_fwd_kvcache(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream) {
    if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || Nq == 0) return FA_OK;
    if (Nk == 0 || (causal && Nk < Nq)) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if ((long long)B * Hq * Nq > (1ll << 30) || (long long)B * Hkv * Nk > (1ll << 31)) return FA_ERR_SHAPE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    // the chunk's rows are the last Nq positions of the key sequence
    return launch_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, causal ? Nk - Nq : 0, d, scale, causal, nullptr,
                      static_cast<cudaStream_t>(stream), ds->status, ds->num_sms, next_sched(ds));
}

extern "C" int fa_fwd_kvcache_varlen(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                     int Hkv, int Nq, int Nk, int d, float scale, int causal,
                                     const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, void* stream) {
    if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || Nq == 0) return FA_OK;
    if (Nk == 0) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
        return FA_ERR_ALIGN;
    if (B > kMaxSeqs) return FA_ERR_SHAPE;
    if ((long long)Hq * Nq > (1ll << 30) || (long long)Hkv * Nk > (1ll << 31)) return FA_ERR_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    return launch_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, 0, d, scale, causal, cu_seqlens_q,
                      static_cast<cudaStream_t>(stream), ds->status, ds->num_sms, next_sched(ds), 0, 1, nullptr,
                      nullptr, false, 1.f, 1.f, cu_seqlens_k);
}

// ------------------------------------------------------------ split keys
// Decode-shaped problems (a few query rows against a long cache) have too few
// 128-row tiles to occupy the GPU.  Two changes fix that.  The query rows of
// the Hq / Hkv heads that share a key/value head are packed into one tile:
// in the [B, Hq, Nq, d] layout they are adjacent, so the problem is read as
// Hkv heads of Hq / Hkv * Nq rows, row r at position Nk - Nq + r % Nq.  And
// the key blocks are cut into splits that run as separate work items, each
// writing its O / l and logsumexp in fp32 to the workspace, merged by
// fa_combine_kernel.
namespace fa_sm100 {

constexpr int kMaxSplits = 256;

struct SplitShape {
    int Hq, Hkv, N, qmod;      // the problem as the kernel sees it
};

static SplitShape split_shape(int Hq, int Hkv, int Nq) {
    const int g = Hq / Hkv;
    if (g > 1 && Nq < kBlockM) return {Hkv, Hkv, g * Nq, Nq};
    return {Hq, Hkv, Nq, 0};
}

static size_t split_workspace_bytes(int B, int Hq, int Nq, int d, int splits) {
    if (splits <= 1) return 0;
    const size_t rows = static_cast<size_t>(B) * Hq * Nq;
    return static_cast<size_t>(splits) * rows * (d + 1) * sizeof(float);
}

// Split count: the one minimising (waves of work items) x (key blocks per
// item + 2 blocks of per-item overhead), smallest on ties.
static int choose_splits(int B, int Hq, int Hkv, int Nq, int Nk, int num_sms) {
    const SplitShape sh = split_shape(Hq, Hkv, Nq);
    const long long units = (long long)B * sh.Hq * ((sh.N + kRowsPerItem - 1) / kRowsPerItem);
    const int nblocks = (Nk + kBlockN - 1) / kBlockN;
    const int smax = std::max(1, std::min(nblocks, kMaxSplits));
    int best = 1;
    double best_cost = 1e300;
    for (int sp = 1; sp <= smax; ++sp) {
        const long long waves = (units * sp + num_sms - 1) / num_sms;
        const double cost = (double)waves * ((nblocks + sp - 1) / sp + 2);
        if (cost < best_cost) {
            best_cost = cost;
            best = sp;
        }
    }
    return best;
}

}  // namespace fa_sm100

extern "C" int fa_splitkv_num_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
    if (B < 1 || Hq < 1 || Nq < 1 || Nk < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    return choose_splits(B, Hq, Hkv, Nq, Nk, ds->num_sms);
}

extern "C" size_t fa_splitkv_workspace_bytes(int B, int Hq, int Nq, int d, int num_splits) {
    if (B < 0 || Hq < 1 || Nq < 0 || (d != 64 && d != 128) || num_splits < 1 || num_splits > kMaxSplits) return 0;
    return split_workspace_bytes(B, Hq, Nq, d, num_splits);
}

extern "C" int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int Nq, int Nk, int d, float scale, int causal, int num_splits,
                              void* workspace, size_t workspace_bytes, void* stream) {
    if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_SHAPE;
    if (B == 0 || Nq == 0) return FA_OK;
    if (Nk == 0 || (causal && Nk < Nq)) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if ((long long)B * Hq * Nq > (1ll << 30) || (long long)B * Hkv * Nk > (1ll << 31)) return FA_ERR_SHAPE;
    if ((long long)B * Hq * Nq * num_splits > (1ll << 31)) return FA_ERR_SHAPE;
    const size_t need = split_workspace_bytes(B, Hq, Nq, d, num_splits);
    if (need > 0) {
        if (!workspace) return FA_ERR_NULL;
        if (!aligned(workspace, 16)) return FA_ERR_ALIGN;
        if (workspace_bytes < need) return FA_ERR_SHAPE;
    }

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const SplitShape sh = split_shape(Hq, Hkv, Nq);
    const int q_off = causal ? Nk - Nq : 0;
    if (num_splits == 1)
        return launch_fwd(q, k, v, o, lse, B, sh.Hq, sh.Hkv, sh.N, Nk, q_off, d, scale, causal, nullptr, s,
                          ds->status, ds->num_sms, next_sched(ds), sh.qmod);
    const long long rows = (long long)B * Hq * Nq;
    float* o_part = static_cast<float*>(workspace);
    float* lse_part = o_part + static_cast<size_t>(num_splits) * rows * d;
    const int rc = launch_fwd(q, k, v, o, lse, B, sh.Hq, sh.Hkv, sh.N, Nk, q_off, d, scale, causal, nullptr, s,
                              ds->status, ds->num_sms, next_sched(ds), sh.qmod, num_splits, o_part, lse_part);
    if (rc != FA_OK) return rc;
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    if (d == 64)
        fa_combine_kernel<64><<<grid, 256, 0, s>>>(o_part, lse_part, static_cast<uint16_t*>(o), lse, rows, num_splits);
    else
        fa_combine_kernel<128><<<grid, 256, 0, s>>>(o_part, lse_part, static_cast<uint16_t*>(o), lse, rows, num_splits);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

static int fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, float scale, int causal, float q_scale, float k_scale, float v_scale,
                   const int32_t* cu_seqlens, void* stream) {
    const bool packed = cu_seqlens != nullptr;
    if (B < 0 || N < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (!(q_scale > 0.f) || !(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(q_scale) ||
        !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return FA_ERR_SHAPE;
    if (B == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if (packed && (B > kMaxSeqs || !aligned(cu_seqlens, 4))) return B > kMaxSeqs ? FA_ERR_SHAPE : FA_ERR_ALIGN;
    if ((packed ? (long long)Hq * N : (long long)B * Hq * N) > (1ll << 30)) return FA_ERR_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    return launch_fwd(q, k, v, o, lse, B, Hq, Hkv, N, N, 0, d, scale, causal, cu_seqlens,
                      static_cast<cudaStream_t>(stream), ds->status, ds->num_sms, next_sched(ds), 0, 1, nullptr,
                      nullptr, true, q_scale * k_scale, v_scale);
}

extern "C" int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int N, int d, float scale, int causal, float q_scale, float k_scale, float v_scale,
                          void* stream) {
    return fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale, nullptr, stream);
}

extern "C" int fa_fwd_fp8_varlen(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                 int Hkv, int N, int d, float scale, int causal, float q_scale, float k_scale,
                                 float v_scale, const int32_t* cu_seqlens, void* stream) {
    if (!cu_seqlens && B > 0 && N > 0) return FA_ERR_NULL;
    return fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale, cu_seqlens, stream);
}

extern "C" int fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B,
                              int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream) {
    if (B < 0 || Nq < 0 || Nk < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || Nq == 0) return FA_OK;
    if (Nk == 0 || (causal && Nk < Nq)) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o_part || !lse_part) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_part, 16) || !aligned(lse_part, 4))
        return FA_ERR_ALIGN;
    if ((long long)B * Hq * Nq > (1ll << 30) || (long long)B * Hkv * Nk > (1ll << 31)) return FA_ERR_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    return launch_fwd(q, k, v, nullptr, nullptr, B, Hq, Hkv, Nq, Nk, causal ? Nk - Nq : 0, d, scale, causal, nullptr,
                      static_cast<cudaStream_t>(stream), ds->status, ds->num_sms, next_sched(ds), 0, 1, o_part,
                      lse_part);
}

extern "C" int fa_merge_partials(const float* o_parts, const float* lse_parts, int nparts, long long rows, int d,
                                 void* o, float* lse, void* stream) {
    if (nparts < 1 || nparts > 4096 || rows < 0) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (rows == 0) return FA_OK;
    if (rows * nparts > (1ll << 40)) return FA_ERR_SHAPE;
    if ((rows + 7) / 8 > 0x7fffffffll) return FA_ERR_SHAPE;     // grid x: 8 rows per block
    if (!o_parts || !lse_parts || !o || !lse) return FA_ERR_NULL;
    if (!aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(o, 16) || !aligned(lse, 4)) return FA_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    if (d == 64)
        fa_combine_kernel<64><<<grid, 256, 0, s>>>(o_parts, lse_parts, static_cast<uint16_t*>(o), lse, rows, nparts);
    else
        fa_combine_kernel<128><<<grid, 256, 0, s>>>(o_parts, lse_parts, static_cast<uint16_t*>(o), lse, rows, nparts);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

extern "C" int fa_selftest_watchdog(int timeout_ms, void* stream) {
    if (timeout_ms < 1 || timeout_ms > 2000) return FA_ERR_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    Params P;
    std::memset(&P, 0, sizeof(P));
    P.status = ds->status;
    P.timeout_ns = static_cast<unsigned long long>(timeout_ms) * 1000000ull;
    fa_watchdog_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(P);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

extern "C" int fa_get_device_status(void* stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    const int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int h[4] = {0, 0, 0, 0};
    if (cudaMemcpyAsync(h, ds->status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_LAUNCH;
    if (cudaMemsetAsync(ds->status, 0, sizeof(h), s) != cudaSuccess) return FA_ERR_LAUNCH;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_LAUNCH;
    return h[0];
}

extern "C" const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_NULL: return "a required pointer is NULL";
        case FA_ERR_SHAPE: return "a size is negative or out of the supported range";
        case FA_ERR_HEADDIM: return "head dimension must be 64 or 128";
        case FA_ERR_GQA: return "Hq must be a positive multiple of Hkv";
        case FA_ERR_ALIGN: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
        case FA_ERR_ARCH: return "current device is not compute capability 10.0 (B200)";
        case FA_ERR_LAUNCH: return "CUDA launch or runtime error";
        case FA_ERR_DEVICE_TIMEOUT: return "device watchdog: a pipeline wait timed out";
        case FA_ERR_SEQLENS: return "cu_seqlens inconsistent with B and N";
        default: return "unknown status";
    }
}

// ======================================================= no-allocation entry
// fa_fwd_noalloc: the same forward for callers that must not allocate device
// memory.  The only global memory fa_fwd uses beyond the caller's buffers is
// its device status word, which fa_fwd allocates with cudaMalloc on its first
// call on a device.  Here that scratch lives in a fixed array compiled into the
// library instead; every GPU that loads the library holds one copy of it
// until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = 256;       // the array's size: the stated maximum
constexpr size_t kStatusBytes = 4 * sizeof(int);   // the status words, at the start of the array
constexpr int kNoAllocSchedSlots = 16;             // work counters after them (64-bit words)
static_assert(kStatusBytes + kNoAllocSchedSlots * sizeof(unsigned long long) <= kNoAllocScratchBytes,
              "no-alloc scratch too small");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocState {
    bool init = false;
    int status_code = FA_OK;
    int num_sms = 0;
    int* scratch = nullptr;    // device address of g_noalloc_scratch on this device
    std::atomic<unsigned> sched_seq{0};
};
NoAllocState g_noalloc[fa_sm100::kMaxDevices];
std::mutex g_noalloc_mu;

// One-time set-up per device, with that device current: properties, the
// tensor-map encoder, the kernels' shared-memory limits, and the device
// address of the scratch array (the array's name is only a host-side handle).
// None of these allocate device memory.
int noalloc_setup(int dev, NoAllocState** out) {
    using namespace fa_sm100;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocState& st = g_noalloc[dev];
    if (!st.init) {
        st.init = true;
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            st.status_code = FA_ERR_LAUNCH;
        } else if (prop.major != 10 || prop.minor != 0) {
            st.status_code = FA_ERR_ARCH;
        } else {
            st.num_sms = prop.multiProcessorCount;
            bool good = true;
            {
                std::lock_guard<std::mutex> lock2(g_mu);
                if (!g_encode) {
                    cudaDriverEntryPointQueryResult q;
                    void* fn = nullptr;
                    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
                        q == cudaDriverEntryPointSuccess)
                        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
                }
                good = g_encode != nullptr;
            }
            void* ptr = nullptr;
            good = good && cudaGetSymbolAddress(&ptr, g_noalloc_scratch) == cudaSuccess && ptr != nullptr;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, false>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<64, true>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, false>::kSmemBytes) == cudaSuccess;
            good = good && cudaFuncSetAttribute(fa_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                Cfg<128, true>::kSmemBytes) == cudaSuccess;
            st.scratch = static_cast<int*>(ptr);
            st.status_code = good ? FA_OK : FA_ERR_LAUNCH;
        }
    }
    *out = &st;
    return st.status_code;
}

}  // namespace

extern "C" int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int N, int d, float scale, int causal, const int32_t* cu_seqlens,
                              void* stream) {
    using namespace fa_sm100;
    const bool packed = cu_seqlens != nullptr;
    if (B < 0 || N < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || N == 0) return FA_OK;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if (packed && (B > kMaxSeqs || !aligned(cu_seqlens, 4))) return B > kMaxSeqs ? FA_ERR_SHAPE : FA_ERR_ALIGN;
    const long long rows = packed ? (long long)Hq * N : (long long)B * Hq * N;
    if (rows > (1ll << 30)) return FA_ERR_SHAPE;
    // the scratch this call needs must fit the fixed array; the status words
    // do not grow with the problem, so only a changed build could fail here
    if (kStatusBytes > kNoAllocScratchBytes) return FA_ERR_SHAPE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    NoAllocState* st = nullptr;
    const int rc = noalloc_setup(dev, &st);
    if (rc != FA_OK) return rc;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status words keep the previous call's contents: start this call at zero
    if (cudaMemsetAsync(st->scratch, 0, kStatusBytes, s) != cudaSuccess) return FA_ERR_LAUNCH;
    const Sched sched = next_sched(st->sched_seq, reinterpret_cast<unsigned long long*>(st->scratch + 4),
                                   kNoAllocSchedSlots);
    return launch_fwd(q, k, v, o, lse, B, Hq, Hkv, N, N, 0, d, scale, causal, cu_seqlens, s, st->scratch,
                      st->num_sms, sched);
}

extern "C" int fa_get_noalloc_status(void* stream) {
    using namespace fa_sm100;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    NoAllocState* st = nullptr;
    const int rc = noalloc_setup(dev, &st);
    if (rc != FA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int h[4] = {0, 0, 0, 0};
    static_assert(sizeof(h) == kStatusBytes, "status words");
    if (cudaMemcpyAsync(h, st->scratch, kStatusBytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_LAUNCH;
    if (cudaMemsetAsync(st->scratch, 0, kStatusBytes, s) != cudaSuccess) return FA_ERR_LAUNCH;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_LAUNCH;
    return h[0];
}
