// fa_bwd.cu -- attention backward (dQ, dK, dV) for B200 (sm_100a) and its C ABI.
//
// The method's backward pass keeps the forward's memory saving: it does not
// store the score matrix, it recomputes the scores block by block from Q and
// K (pages: "Flash Attention", 14cs17.netlify.app, "Common Pitfalls",
// Pitfall 3; fromzero2ai.dev, "Core Mechanisms of FlashAttention", item 3).
// The gradients are those of the forward's definition: with
// P = softmax(scale Q K^T) (masked), O = P V and the upstream gradient dO,
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D_i = sum_j dO_ij O_ij,
//     dQ = scale dS K,  dK = scale dS^T Q,
// and P_ij = exp(scale q_i.k_j - lse_i) from the logsumexp the forward saved.
//
// Three kernels on the caller's stream:
//   1. fa_bwd_prep_kernel: D_i = rowsum(dO * O) and lse_i * log2(e) per query
//      row, in row-padded fp32 arrays, and the fp32 dQ accumulator cleared.
//   2. fa_bwd_kernel: one persistent CTA per SM; a work item is one 128-key
//      block K_j, V_j of one (batch, kv head).  It keeps dK_j and dV_j in TMEM
//      while it walks the query blocks Q_i, dO_i of every query head of the
//      group (under the causal mask, i >= j only); per block it recomputes
//      S^T = K_j Q_i^T, forms P^T and dS^T, accumulates dV_j and dK_j, and
//      adds dQ_i's share into the fp32 accumulator with vector reductions.
//   3. fa_bwd_dq_kernel: dQ = scale * accumulator, rounded to bf16.
//
// fa_bwd_kernel roles (512 threads):
//   warps 0-7   two P/dS warpgroups, one thread per key row, warpgroup g
//               taking query columns 64g .. 64g+63: tcgen05.ld of S^T,
//               P^T = exp2(S^T scale log2e - lse log2e) (masked), bf16 P^T
//               back into TMEM; then tcgen05.ld of dP^T, dS^T = P^T (dP^T - D)
//               to shared memory (bf16, 128-byte swizzled K-major tile).
//   warps 8-11  dQ warpgroup, one thread per query row: tcgen05.ld of the
//               block's dQ_i share, staged through shared memory so that each
//               red.global.add.v4.f32 instruction covers whole 128-byte rows
//               of the accumulator; at the end of an item, dK_j and dV_j from
//               TMEM to HBM (bf16).
//   warp 13     MMA issuer (one thread); warps 14 and 15 TMA producers (one
//               thread each: K, V, Q and the lse / D slices; dO);
//   warp 12     TMEM allocation.
//
// TMEM columns (512): X [0,128) S^T, then P^T (bf16) in [0,64);
// Y [128,256) dP^T, then the block's dQ_i share; dV [256,256+D); dK [384,384+D).
// Shared memory: K_j, V_j, two Q slots (with their lse and D slices), one dO
// slot, the dS tile and the dQ staging tiles.
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
namespace bwd {

// Optional pipeline timeline (compile with -DFA_TRACE): CTA 0 records clock64
// stamps as [role][iteration][event], 256 iterations and 8 events per role;
// the buffer is set with fa_bwd_trace_set.
#ifdef FA_TRACE
__device__ unsigned long long* g_btrace = nullptr;
#define BWD_TRACE(role, it, ev)                                                                          \
    do {                                                                                                 \
        if (blockIdx.x == 0 && g_btrace && (it) < 256) g_btrace[((role) * 256 + (it)) * 8 + (ev)] = clock64(); \
    } while (0)
#else
#define BWD_TRACE(role, it, ev) \
    do {                        \
    } while (0)
#endif

constexpr int kBlock = 128;            // keys per item, queries per step
constexpr int kMaxSeqsBwd = 1024;      // packed batches: sequences (one CTA builds the tables)
constexpr int kThreads = 512;
constexpr int kDqWarp0 = 8;            // warps 8-11: dQ warpgroup
constexpr int kAllocWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kLoadWarp = 14;
// setmaxnreg split of the 512 x 128 registers: 2 x 128 x 144 (P/dS) +
// 128 x 160 (dQ) + 128 x 64 (control) = 512 x 128
constexpr uint32_t kPdsRegs = 144;
constexpr uint32_t kDqRegs = 160;
constexpr uint32_t kOtherRegs = 64;
constexpr uint32_t kTmemCols = 512;
constexpr int kBoxBytes = kBlock * 64 * 2;   // one 128-row x 64-column bf16 TMA box
constexpr uint32_t kColX = 0, kColY = 128, kColDV = 256, kColDK = 384;

enum WaitSite : int {
    kSiteKvEmpty = 11, kSiteKvFull, kSiteQEmpty, kSiteQFull, kSiteDoEmpty, kSiteDoFull, kSiteS, kSiteP, kSiteDp,
    kSiteDs, kSiteDsFree, kSiteDq, kSiteYFree, kSiteAccDone, kSiteAccFree, kSiteAlign
};

struct alignas(64) Params {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;
    // Per-row vectors and the dQ accumulator live on padded rows: dense,
    // [B, Hq, Npad] with Npad = N rounded up to 128; packed, [Hq, Npad] with
    // sequence s at rows pad_off[s] .. (128-aligned; Npad bounds the total).
    const float* lse2;      // lse * log2(e); +inf on padding rows
    const float* Dvec;      // rowsum(dO * O); 0 on padding rows
    float* dq_acc;          // [.., d] fp32, cleared by the prep kernel
    const int32_t* cu;      // packed: cu_seqlens (B+1 offsets); dense: NULL
    const int* tab;         // packed: work-unit starts [B+1], order [B], pad_off [B+1], total units
    uint16_t* dk;           // dense [B, Hkv, N, d]; packed [N, Hkv, d]; bf16
    uint16_t* dv;           // [B, Hkv, N, d] bf16
    int* status;
    int B, Hq, Hkv, N, Npad, group, causal, packed;
    float scale_log2, scale;
    unsigned long long timeout_ns;
};

struct Misc {
    uint64_t kv_full, kv_empty, q_full[2], q_empty[2], do_full, do_empty;
    uint64_t s_full, p_full, dp_full, ds_full, ds_free, dq_full, y_free, acc_done, acc_free, drain;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kBoxes = D / 64;
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kTileBytes;
    static constexpr int kQOff = kVOff + kTileBytes;              // two slots
    static constexpr int kDoOff = kQOff + 2 * kTileBytes;         // one slot
    static constexpr int kDsOff = kDoOff + kTileBytes;            // 128 x 128 bf16
    static constexpr int kVecOff = kDsOff + kBlock * kBlock * 2;  // lse2[2][128], D[2][128]
    static constexpr int kStageOff = kVecOff + 4 * kBlock * 4;    // dQ staging: 4 warps x 32 rows x 128 B
    static constexpr int kMiscOff = kStageOff + 4 * 32 * 128;
    static constexpr int kLayoutBytes = kMiscOff + (int)sizeof(Misc);
    static_assert(kLayoutBytes <= 232448, "shared memory");
    // the tiles need a 1024-byte aligned base: request room for the padding
    // where it fits; the kernel checks that the padding it needs fits
    static constexpr int kSmemBytes = kLayoutBytes + 1024 <= 232448 ? kLayoutBytes + 1024 : 232448;
};

// One work item: key block j of one (batch or sequence, kv head).
struct Item {
    int b, hk, j;
    int i0;       // first query block (causal: j)
    int nq;       // query blocks per head
    int niter;    // group * (nq - i0)
    int len;      // tokens of the sequence
    int tok0;     // packed: first token of the sequence
    int padoff;   // packed: first padded row of the sequence
};

// Padded row of the per-row vectors and of the dQ accumulator for query head
// h, query block i of the item (dense: [B, Hq, Npad]; packed: [Hq, Npad]).
__device__ __forceinline__ size_t vrow(const Item& it, const Params& p, int h, int i) {
    const size_t base = p.packed ? static_cast<size_t>(h) * p.Npad + it.padoff
                                 : (static_cast<size_t>(it.b) * p.Hq + h) * p.Npad;
    return base + static_cast<size_t>(i) * kBlock;
}

__device__ __forceinline__ int item_of_round(int r) {
    const int G = gridDim.x;
    return r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

// Work units: key blocks j and nk-1-j of one (batch, kv head), run one after
// the other by one CTA.  Under the causal mask block j visits nk - j query
// blocks, so every pair visits nk + 1 (the middle block of an odd count is
// alone).  Units are numbered (batch, kv head)-major, so the CTAs running at
// the same time share few heads and those heads' dQ accumulators stay in L2.
__device__ __forceinline__ int num_work_units(const Params& p) {
    if (p.packed) return p.tab[3 * p.B + 2];
    const int nk = (p.N + kBlock - 1) / kBlock;
    return ((nk + 1) / 2) * p.B * p.Hkv;
}

// Slot r of this CTA's sequence: element r % 2 of work unit
// item_of_round(r / 2).  Returns 0 past the last unit, 2 for the missing
// second element of a lone middle block, 1 with `it` filled in.
__device__ __forceinline__ int next_item(int r, const Params& p, int total_wu, Item& it) {
    const int w = item_of_round(r >> 1);
    if (w >= total_wu) return 0;
    int nk, pr;
    if (!p.packed) {
        nk = (p.N + kBlock - 1) / kBlock;
        const int npairs = (nk + 1) / 2;
        const int u = w / npairs;
        pr = w - u * npairs;
        it.b = u / p.Hkv;
        it.hk = u - it.b * p.Hkv;
        it.len = p.N;
        it.tok0 = 0;
        it.padoff = 0;
    } else {
        // packed: units of sequence order[k] start at wu[k] (longest first)
        const int* wu = p.tab;
        const int* order = p.tab + p.B + 1;
        const int* pad = p.tab + 2 * p.B + 1;
        int lo = 0, hi = p.B - 1;                  // largest k with wu[k] <= w
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (wu[mid] <= w) lo = mid; else hi = mid - 1;
        }
        const int sq = order[lo];
        it.b = sq;
        it.tok0 = p.cu[sq];
        it.len = p.cu[sq + 1] - it.tok0;
        it.padoff = pad[sq];
        nk = (it.len + kBlock - 1) / kBlock;
        const int npairs = (nk + 1) / 2;
        const int rem = w - wu[lo];
        it.hk = rem / npairs;
        pr = rem - it.hk * npairs;
    }
    const int j = (r & 1) ? nk - 1 - pr : pr;
    if ((r & 1) && j == pr) return 2;
    it.j = j;
    it.nq = nk;
    it.i0 = p.causal ? j : 0;
    it.niter = p.group * (it.nq - it.i0);
    return 1;
}

// Iteration n of an item: query head h (of the group) and query block i.
// The query blocks of a head are walked from a starting point that depends
// on the key block, so that CTAs working on the same head at the same time
// add into different rows of the dQ accumulator.
__device__ __forceinline__ void iter_of(const Item& it, int n, const Params& p, int& h, int& i) {
    const int per = it.nq - it.i0;
    const int g = n / per;
    h = it.hk * p.group + g;
    int t = n - g * per + (it.j * 7) % per;
    if (t >= per) t -= per;
    i = it.i0 + t;
}

#ifndef FA_SUSPEND_NS
#define FA_SUSPEND_NS 20000u
#endif

// Bounded wait: gives up after timeout_ns (recording the site in the status
// word and raising the CTA's abort flag) or as soon as another role aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Params& p, Misc& ms, int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, FA_SUSPEND_NS)) return true;
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
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, const Params& p) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > p.timeout_ns) return;
    }
}

// ---------------------------------------------------------------- producer
// Two producer threads: `which` 0 loads K_j, V_j per item and Q_i with its
// lse and D slices per iteration; `which` 1 loads dO_i.  Each runs ahead as
// far as its own buffer slots allow.
template <int D>
__device__ void load_role(const Params& p, Misc& ms, uint8_t* smem, int total, int which) {
    using C = Cfg<D>;
    const uint64_t pol_keep = policy_evict_last();
    const uint32_t s_k = smem_u32(smem + C::kKOff), s_v = smem_u32(smem + C::kVOff);
    const uint32_t s_q = smem_u32(smem + C::kQOff), s_do = smem_u32(smem + C::kDoOff);
    const uint32_t s_vec = smem_u32(smem + C::kVecOff);
    uint32_t item_n = 0, ng = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
        Item it;
        const int st = next_item(r, p, total, it);
        if (st == 0) break;
        if (st == 2) continue;
        if (which == 0) {
            if (!(ok = wait_bar(smem_u32(&ms.kv_empty), (item_n & 1) ^ 1, p, ms, kSiteKvEmpty))) break;
            mbar_arrive_expect_tx(smem_u32(&ms.kv_full), 2 * C::kTileBytes);
            for (int bx = 0; bx < C::kBoxes; ++bx) {
                if (!p.packed) {
                    tma_load_4d(s_k + bx * kBoxBytes, &p.tm_k, smem_u32(&ms.kv_full), bx * 64, it.j * kBlock, it.hk,
                                it.b, pol_keep);
                    tma_load_4d(s_v + bx * kBoxBytes, &p.tm_v, smem_u32(&ms.kv_full), bx * 64, it.j * kBlock, it.hk,
                                it.b, pol_keep);
                } else {
                    tma_load_4d(s_k + bx * kBoxBytes, &p.tm_k, smem_u32(&ms.kv_full), bx * 64, it.hk,
                                it.tok0 + it.j * kBlock, 0, pol_keep);
                    tma_load_4d(s_v + bx * kBoxBytes, &p.tm_v, smem_u32(&ms.kv_full), bx * 64, it.hk,
                                it.tok0 + it.j * kBlock, 0, pol_keep);
                }
            }
            ++item_n;
        }
        for (int n = 0; n < it.niter && ok; ++n, ++ng) {
            int h, i;
            iter_of(it, n, p, h, i);
            const uint32_t slot = ng & 1;
            if (which == 0) {
                // Q_i with its lse and D slices
                BWD_TRACE(3, ng, 0);
                if (!(ok = wait_bar(smem_u32(&ms.q_empty[slot]), ((ng >> 1) & 1) ^ 1, p, ms, kSiteQEmpty))) break;
                BWD_TRACE(3, ng, 1);
                const uint32_t qbar = smem_u32(&ms.q_full[slot]);
                mbar_arrive_expect_tx(qbar, C::kTileBytes + 2 * kBlock * 4);
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                    if (!p.packed)
                        tma_load_4d(s_q + slot * C::kTileBytes + bx * kBoxBytes, &p.tm_q, qbar, bx * 64, i * kBlock, h,
                                    it.b, pol_keep);
                    else
                        tma_load_4d(s_q + slot * C::kTileBytes + bx * kBoxBytes, &p.tm_q, qbar, bx * 64, h,
                                    it.tok0 + i * kBlock, 0, pol_keep);
                }
                const size_t row0 = vrow(it, p, h, i);
                bulk_load(s_vec + slot * kBlock * 4, p.lse2 + row0, kBlock * 4, qbar);
                bulk_load(s_vec + (2 + slot) * kBlock * 4, p.Dvec + row0, kBlock * 4, qbar);
            } else {
                // dO_i
                if (!(ok = wait_bar(smem_u32(&ms.do_empty), (ng & 1) ^ 1, p, ms, kSiteDoEmpty))) break;
                BWD_TRACE(3, ng, 2);
                const uint32_t dbar = smem_u32(&ms.do_full);
                mbar_arrive_expect_tx(dbar, C::kTileBytes);
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                    if (!p.packed)
                        tma_load_4d(s_do + bx * kBoxBytes, &p.tm_do, dbar, bx * 64, i * kBlock, h, it.b, pol_keep);
                    else
                        tma_load_4d(s_do + bx * kBoxBytes, &p.tm_do, dbar, bx * 64, h, it.tok0 + i * kBlock, 0, pol_keep);
                }
            }
        }
    }
    if (!ok) {
        // let the copies already issued land before the CTA goes away: the
        // last item's K/V and the last two slots' loads
        if (which == 0 && item_n > 0) drain_bar(smem_u32(&ms.kv_full), (item_n - 1) & 1, p);
        if (which == 0) {
            for (uint32_t g = (ng > 2 ? ng - 2 : 0); g < ng; ++g) drain_bar(smem_u32(&ms.q_full[g & 1]), (g >> 1) & 1, p);
        } else if (ng > 0) {
            drain_bar(smem_u32(&ms.do_full), (ng - 1) & 1, p);
        }
    }
}

// ------------------------------------------------------------- MMA issuer
template <int D>
__device__ __forceinline__ void mma_qk(uint32_t d_tmem, uint64_t a, uint64_t b) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBlock, kBlock, false);
    if constexpr (D == 128)
        umma_ss_k128_x8(d_tmem, a, b, idesc);
    else
        umma_ss_k64_x4(d_tmem, a, b, idesc);
}

// The MMA issuer: all 32 lanes of the warp run the loop (waits included); one
// elected lane issues each batch of MMAs and commits.
template <int D>
__device__ void mma_role(const Params& p, Misc& ms, uint8_t* smem, uint32_t tmem, int total) {
    using C = Cfg<D>;
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    // K-major views (inner dimension d inside the swizzled rows)
    const uint64_t dk_k = smem_desc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
    const uint64_t dv_k = smem_desc_sw128(smem_u32(smem + C::kVOff), 16, 1024);
    const uint64_t dq_k0 = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
    const uint64_t ddo_k0 = smem_desc_sw128(smem_u32(smem + C::kDoOff), 16, 1024);
    const uint64_t dds_k = smem_desc_sw128(smem_u32(smem + C::kDsOff), 16, 1024);
    // MN-major views (rows are the reduction dimension)
    const uint64_t dk_mn = smem_desc_sw128(smem_u32(smem + C::kKOff), kBoxBytes, 1024);
    const uint64_t dq_mn0 = smem_desc_sw128(smem_u32(smem + C::kQOff), kBoxBytes, 1024);
    const uint64_t ddo_mn0 = smem_desc_sw128(smem_u32(smem + C::kDoOff), kBoxBytes, 1024);
    const uint64_t dds_mn = smem_desc_sw128(smem_u32(smem + C::kDsOff), kBoxBytes, 1024);
    constexpr uint32_t id_dv = idesc_bf16_f32(kBlock, D, true);          // P^T (TMEM) x dO (MN)
    constexpr uint32_t id_dk = idesc_bf16_f32(kBlock, D, true);          // dS^T (K-major) x Q (MN)
    constexpr uint32_t id_dq = idesc_bf16_f32(kBlock, D, true, true);    // dS (MN) x K (MN)
    uint32_t item_n = 0, ng = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
        Item it;
        const int st = next_item(r, p, total, it);
        if (st == 0) break;
        if (st == 2) continue;
        if (!(ok = wait_all(smem_u32(&ms.kv_full), item_n & 1, p, ms, kSiteKvFull))) break;
        tc_fence_after();
        for (int n = 0; n < it.niter && ok; ++n, ++ng) {
            const uint32_t slot = ng & 1;
            if (n == 0) {          // S^T of the item's first block
                if (!(ok = wait_all(smem_u32(&ms.q_full[slot]), (ng >> 1) & 1, p, ms, kSiteQFull))) break;
                tc_fence_after();
                if (elect_one()) {
                    mma_qk<D>(tmem + kColX, dk_k, dq_k0 + slot * kTileStep);
                    umma_commit(smem_u32(&ms.s_full));
                }
                __syncwarp();
            }
            // dP^T = V_j dO_i^T (once the previous dQ share has left Y) and
            // dV_j += P^T dO_i (once P^T is in TMEM), whichever is ready first
            BWD_TRACE(0, ng, 0);
            if (!(ok = wait_all(smem_u32(&ms.do_full), ng & 1, p, ms, kSiteDoFull))) break;
            BWD_TRACE(0, ng, 1);
            const uint64_t ddo_k = ddo_k0, ddo_mn = ddo_mn0;
            bool dp_issued = false;
            if (__all_sync(0xffffffffu, mbar_try_wait(smem_u32(&ms.y_free), (ng & 1) ^ 1))) {
                tc_fence_after();
                if (elect_one()) {
                    mma_qk<D>(tmem + kColY, dv_k, ddo_k);
                    umma_commit(smem_u32(&ms.dp_full));
                }
                __syncwarp();
                dp_issued = true;
            }
            if (!(ok = wait_all(smem_u32(&ms.p_full), ng & 1, p, ms, kSiteP))) break;
            BWD_TRACE(0, ng, 2);
            if (n == 0 && !(ok = wait_all(smem_u32(&ms.acc_free), (item_n & 1) ^ 1, p, ms, kSiteAccFree))) break;
            tc_fence_after();
            if (elect_one()) umma_ts_kv128_x8(tmem + kColDV, tmem + kColX, ddo_mn, id_dv, n > 0 ? 1u : 0u);
            __syncwarp();
            if (!dp_issued) {
                if (!(ok = wait_all(smem_u32(&ms.y_free), (ng & 1) ^ 1, p, ms, kSiteYFree))) break;
                tc_fence_after();
                if (elect_one()) {
                    mma_qk<D>(tmem + kColY, dv_k, ddo_k);
                    umma_commit(smem_u32(&ms.dp_full));
                }
                __syncwarp();
            }
            if (elect_one()) umma_commit(smem_u32(&ms.do_empty));
            __syncwarp();
            BWD_TRACE(0, ng, 3);
            // S^T of the next block (X is free once dV has read P^T: in order)
            if (n + 1 < it.niter) {
                const uint32_t ns = (ng + 1) & 1;
                if (!(ok = wait_all(smem_u32(&ms.q_full[ns]), ((ng + 1) >> 1) & 1, p, ms, kSiteQFull))) break;
                tc_fence_after();
                if (elect_one()) {
                    mma_qk<D>(tmem + kColX, dk_k, dq_k0 + ns * kTileStep);
                    umma_commit(smem_u32(&ms.s_full));
                }
                __syncwarp();
            }
            // dK_j += dS^T Q_i and dQ_i share = dS K_j, once dS is in shared memory
            BWD_TRACE(0, ng, 4);
            if (!(ok = wait_all(smem_u32(&ms.ds_full), ng & 1, p, ms, kSiteDs))) break;
            BWD_TRACE(0, ng, 5);
            tc_fence_after();
            // dQ first: the dQ warpgroup can start reading Y while dK runs
            if (elect_one()) {
                umma_ss_mnA_mnB_k128_x8(tmem + kColY, dds_mn, dk_mn, id_dq);
                umma_commit(smem_u32(&ms.dq_full));
                umma_ss_kA_mnB_k128_x8(tmem + kColDK, dds_k, dq_mn0 + slot * kTileStep, id_dk, n > 0 ? 1u : 0u);
                umma_commit(smem_u32(&ms.ds_free));
                umma_commit(smem_u32(&ms.q_empty[slot]));
            }
            __syncwarp();
            BWD_TRACE(0, ng, 6);
            if (dp_issued) BWD_TRACE(0, ng, 7);
            if (n == it.niter - 1 && elect_one()) {
                umma_commit(smem_u32(&ms.acc_done));
                umma_commit(smem_u32(&ms.kv_empty));
            }
            __syncwarp();
        }
        ++item_n;
    }
    __syncwarp();
    if (elect_one()) umma_commit(smem_u32(&ms.drain));
    __syncwarp();
    drain_bar(smem_u32(&ms.drain), 0, p);
}

// -------------------------------------------------- P / dS warpgroup
// Byte offset of 16-byte chunk `c16` (8 bf16 columns, 0..15) of row `r` in a
// 128-row x 128-column bf16 tile stored as two 128-byte-swizzled 64-column
// boxes (the layout TMA writes, read K-major or MN-major by the MMAs).
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c16) {
    return static_cast<uint32_t>((c16 >> 3) * kBoxBytes + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}

template <int D>
__device__ void pds_role(const Params& p, Misc& ms, uint8_t* smem, uint32_t tmem, int warp, int lane, int total) {
    using C = Cfg<D>;
    const int g = warp / 4;                              // warpgroup: query columns 64g .. 64g+63
    const int wq = warp % 4;                             // TMEM lane quarter
    const int r = wq * 32 + lane;                        // key row inside the block
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tx = tmem + lane_off + kColX, ty = tmem + lane_off + kColY;
    const uint32_t vec = smem_u32(smem + C::kVecOff);
    const uint32_t ds_tile = smem_u32(smem + C::kDsOff);
    const float sl2 = p.scale_log2;
    uint32_t ng = 0;
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
        Item it;
        const int st = next_item(rr, p, total, it);
        if (st == 0) break;
        if (st == 2) continue;
        const bool key_valid = it.j * kBlock + r < it.len;
        for (int n = 0; n < it.niter; ++n, ++ng) {
            int h, i;
            iter_of(it, n, p, h, i);
            const uint32_t slot = ng & 1;
            const uint32_t lse2 = vec + (slot * kBlock + 64 * g) * 4;
            const uint32_t dvec = vec + ((2 + slot) * kBlock + 64 * g) * 4;
            if (r == 0 && g == 0) BWD_TRACE(1, ng, 0);
            ok = wait_bar(smem_u32(&ms.s_full), ng & 1, p, ms, kSiteS);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[64];
            {
                uint32_t (&sa)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
                uint32_t (&sb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
                tmem_ld64_sync(tx + 64 * g, sa, sb);
            }
            // P^T = exp2(S^T * scale * log2 e - lse * log2 e) for key r and query
            // 64g + c; masked: query < key on the diagonal block, and every
            // query of a key row past the sequence end
            const int cmin = !key_valid ? 64 : ((p.causal && i == it.j) ? r - 64 * g : 0);
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                float4 l4[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) l4[t] = lds_f4(lse2 + (c0 + 4 * t) * 4);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const int c = c0 + 4 * t;
                    const float e0 = ex2_approx(fmaf(__uint_as_float(s[c]), sl2, -l4[t].x));
                    const float e1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), sl2, -l4[t].y));
                    const float e2 = ex2_approx(fmaf(__uint_as_float(s[c + 2]), sl2, -l4[t].z));
                    const float e3 = ex2_approx(fmaf(__uint_as_float(s[c + 3]), sl2, -l4[t].w));
                    s[c] = __float_as_uint(c < cmin ? 0.f : e0);
                    s[c + 1] = __float_as_uint(c + 1 < cmin ? 0.f : e1);
                    s[c + 2] = __float_as_uint(c + 2 < cmin ? 0.f : e2);
                    s[c + 3] = __float_as_uint(c + 3 < cmin ? 0.f : e3);
                }
            }
            {
                uint32_t pk[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(__uint_as_float(s[2 * t]), __uint_as_float(s[2 * t + 1]));
                tmem_st32(tx + 32 * g, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ms.p_full));
            if (r == 0 && g == 0) BWD_TRACE(1, ng, 3);
            // dS^T = P^T (dP^T - D), into box g of the shared dS tile
            ok = wait_bar(smem_u32(&ms.dp_full), ng & 1, p, ms, kSiteDp);
            if (r == 0 && g == 0) BWD_TRACE(1, ng, 4);
            ok = ok && wait_bar(smem_u32(&ms.ds_free), (ng & 1) ^ 1, p, ms, kSiteDsFree);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            if (r == 0 && g == 0) BWD_TRACE(1, ng, 5);
            tc_fence_after();
#pragma unroll
            for (int q4 = 0; q4 < 2; ++q4) {
                uint32_t dp[32];
                tmem_ld32_sync(ty + 64 * g + 32 * q4, dp);
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    float4 d4[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) d4[t] = lds_f4(dvec + (32 * q4 + 16 * hq + 4 * t) * 4);
                    uint32_t pk[8];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int c = 32 * q4 + 16 * hq + 4 * t;
                        const int e = 16 * hq + 4 * t;
                        pk[2 * t] = pack_bf16x2(__uint_as_float(s[c]) * (__uint_as_float(dp[e]) - d4[t].x),
                                                __uint_as_float(s[c + 1]) * (__uint_as_float(dp[e + 1]) - d4[t].y));
                        pk[2 * t + 1] = pack_bf16x2(__uint_as_float(s[c + 2]) * (__uint_as_float(dp[e + 2]) - d4[t].z),
                                                    __uint_as_float(s[c + 3]) * (__uint_as_float(dp[e + 3]) - d4[t].w));
                    }
                    const int c16 = 8 * g + 4 * q4 + 2 * hq;
                    sts_u4(ds_tile + sw128_chunk(r, c16), pk[0], pk[1], pk[2], pk[3]);
                    sts_u4(ds_tile + sw128_chunk(r, c16 + 1), pk[4], pk[5], pk[6], pk[7]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ms.ds_full));
            if (r == 0 && g == 0) BWD_TRACE(1, ng, 6);
        }
    }
}

// ------------------------------------------------------- dQ warpgroup
template <int D>
__device__ void dq_role(const Params& p, Misc& ms, uint8_t* smem, uint32_t tmem, int wq, int lane, int total) {
    using C = Cfg<D>;
    const int r = wq * 32 + lane;                       // query row (dQ) or key row (dK, dV)
    // this warp's 32 x 32 fp32 staging tile: 128-byte rows, 16-byte chunks
    // XOR-swizzled by row; rows go in by thread and come out by row
    const uint32_t stage = smem_u32(smem + C::kStageOff) + wq * 32 * 128;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t ty = tmem + lane_off + kColY;
    uint32_t item_n = 0, ng = 0;
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
        Item it;
        const int st = next_item(rr, p, total, it);
        if (st == 0) break;
        if (st == 2) continue;
        for (int n = 0; n < it.niter; ++n, ++ng) {
            int h, i;
            iter_of(it, n, p, h, i);
            if (r == 0) BWD_TRACE(2, ng, 0);
            ok = wait_bar(smem_u32(&ms.dq_full), ng & 1, p, ms, kSiteDq);
            if (r == 0) BWD_TRACE(2, ng, 1);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            // row r of the block's dQ share: into registers first, so that Y can
            // take the next dP before the reductions go out
            float* dst = p.dq_acc + (vrow(it, p, h, i) + r) * D;
            uint32_t v[D];
            if constexpr (D == 128) {
                tmem_ld128_sync(ty, v);
            } else {
                uint32_t (&va)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
                uint32_t (&vb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
                tmem_ld64_sync(ty, va, vb);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ms.y_free));
            if (r == 0) BWD_TRACE(2, ng, 2);
            // 32 columns at a time through the staging tile: each reduction
            // instruction of the warp then covers 4 rows x 128 bytes
            float* dst0 = dst - static_cast<size_t>(lane) * D;          // row wq*32 of the share
            const int rsub = lane >> 3, k = lane & 7;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    sts_u4(stage + lane * 128 + ((t ^ (lane & 7)) << 4), v[32 * c + 4 * t], v[32 * c + 4 * t + 1],
                           v[32 * c + 4 * t + 2], v[32 * c + 4 * t + 3]);
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const int row = 4 * rr + rsub;
                    const float4 x = lds_f4(stage + row * 128 + ((k ^ (row & 7)) << 4));
                    red_add_v4(dst0 + static_cast<size_t>(row) * D + 32 * c + 4 * k, x.x, x.y, x.z, x.w);
                }
                __syncwarp();
            }
            if (r == 0) BWD_TRACE(2, ng, 3);
        }
        if (!ok) break;
        // dK_j, dV_j of the item: TMEM -> bf16 -> HBM
        ok = wait_bar(smem_u32(&ms.acc_done), item_n & 1, p, ms, kSiteAccDone);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        ++item_n;
        tc_fence_after();
        const int key = it.j * kBlock + r;
        const size_t row = p.packed ? static_cast<size_t>(it.tok0 + key) * p.Hkv + it.hk
                                    : (static_cast<size_t>(it.b) * p.Hkv + it.hk) * p.N + key;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const float mul = which == 0 ? 1.f : p.scale;
            uint16_t* out = (which == 0 ? p.dv : p.dk) + row * D;
            const uint32_t col = which == 0 ? kColDV : kColDK;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32_sync(tmem + lane_off + col + 32 * c, v);
                uint32_t pk[16];
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    pk[t] = pack_bf16x2(__uint_as_float(v[2 * t]) * mul, __uint_as_float(v[2 * t + 1]) * mul);
                if (key < it.len) {
                    uint4* o4 = reinterpret_cast<uint4*>(out + 32 * c);
#pragma unroll
                    for (int t = 0; t < 4; ++t) o4[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ms.acc_free));
    }
}

// ------------------------------------------------------------------ kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1) fa_bwd_kernel(const __grid_constant__ Params p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (smem - smem_raw > C::kSmemBytes - C::kLayoutBytes) {
        // the launch's shared memory cannot hold the aligned layout: report, do nothing
        if (threadIdx.x == 0 && atomicCAS(p.status, 0, FA_ERR_LAUNCH) == 0) {
            p.status[1] = kSiteAlign;
            p.status[2] = blockIdx.x;
        }
        return;
    }
    Misc& ms = *reinterpret_cast<Misc*>(smem + C::kMiscOff);
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    if (tid == 0) {
        mbar_init(smem_u32(&ms.kv_full), 1);
        mbar_init(smem_u32(&ms.kv_empty), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ms.q_full[s]), 1);
            mbar_init(smem_u32(&ms.q_empty[s]), 1);
        }
        mbar_init(smem_u32(&ms.do_full), 1);
        mbar_init(smem_u32(&ms.do_empty), 1);
        mbar_init(smem_u32(&ms.s_full), 1);
        mbar_init(smem_u32(&ms.p_full), 8);       // one arrival per warp of the two P/dS warpgroups
        mbar_init(smem_u32(&ms.dp_full), 1);
        mbar_init(smem_u32(&ms.ds_full), 8);
        mbar_init(smem_u32(&ms.ds_free), 1);
        mbar_init(smem_u32(&ms.dq_full), 1);
        mbar_init(smem_u32(&ms.y_free), 4);       // one arrival per warp of the dQ warpgroup
        mbar_init(smem_u32(&ms.acc_done), 1);
        mbar_init(smem_u32(&ms.acc_free), 4);
        mbar_init(smem_u32(&ms.drain), 1);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tensormap(&p.tm_q);
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
        prefetch_tensormap(&p.tm_do);
    }
    if (warp == kAllocWarp) {
        tmem_alloc(smem_u32(&ms.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    const int total = num_work_units(p);

    if (warp < kDqWarp0) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPdsRegs));
        pds_role<D>(p, ms, smem, tmem, warp, lane, total);
    } else if (warp < kDqWarp0 + 4) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDqRegs));
        dq_role<D>(p, ms, smem, tmem, warp - kDqWarp0, lane, total);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
        if (warp == kMmaWarp) {
            mma_role<D>(p, ms, smem, tmem, total);      // all 32 lanes
            __syncwarp();
        } else if (warp == kLoadWarp) {
            if (lane == 0) load_role<D>(p, ms, smem, total, 0);
            __syncwarp();
        } else if (warp == kLoadWarp + 1) {
            if (lane == 0) load_role<D>(p, ms, smem, total, 1);
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

// Packed batches: checks cu_seqlens and builds the schedule tables (one CTA
// of 1024 threads, B <= 1024): the sequences ordered by key-block count
// (longest first), the first work unit of each in that order, and the first
// padded row of each sequence (rows rounded up to 128 per sequence).  Bad
// offsets record FA_ERR_SEQLENS and leave no work.
__global__ void __launch_bounds__(1024) fa_bwd_tables_kernel(const int32_t* __restrict__ cu, int B, int N, int Hkv,
                                                             int* tab, int* status) {
    __shared__ int nk[1024];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = (cu[0] != 0 || cu[B] != N) ? 1 : 0;
    __syncthreads();
    if (tid < B) {
        const int L = cu[tid + 1] - cu[tid];
        if (L < 0) atomicOr(&bad, 1);
        nk[tid] = L > 0 ? (L + kBlock - 1) / kBlock : 0;
    }
    __syncthreads();
    int* wu = tab;
    int* order = tab + B + 1;
    int* pad = tab + 2 * B + 1;
    if (tid < B) {
        int rank = 0;
        for (int u = 0; u < B; ++u) rank += (nk[u] > nk[tid]) || (nk[u] == nk[tid] && u < tid);
        order[rank] = tid;
    }
    __syncthreads();
    if (tid == 0) {
        wu[0] = 0;
        for (int k = 0; k < B; ++k) wu[k + 1] = wu[k] + ((nk[order[k]] + 1) / 2) * Hkv;
        pad[0] = 0;
        for (int q = 0; q < B; ++q) pad[q + 1] = pad[q] + nk[q] * kBlock;
        tab[3 * B + 2] = bad ? 0 : wu[B];
        tab[3 * B + 3] = bad ? -1 : pad[B];       // -1: offsets rejected
        if (bad) atomicCAS(status, 0, FA_ERR_SEQLENS);
    }
}

// Largest s in [0, n) with a[s] <= x (a non-decreasing, a[0] <= x).
__device__ __forceinline__ int last_le(const int* a, int n, long long x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// D_i = sum_c dO_ic O_ic (fp32 from bf16), lse_i * log2(e), on the padded
// rows (padding: D = 0, lse2 = +inf so that P = 0 there); and the dQ
// accumulator cleared.  One warp per padded row.  Dense: rows [B, Hq, Npad],
// O / dO [B, Hq, N, d], lse [B, Hq, N].  Packed: rows [Hq, Npad], O / dO
// [N, Hq, d], lse [Hq, N].
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                          const float* __restrict__ lse, float* lse2, float* Dvec,
                                                          float* dq_acc, int N, int Npad, long long rows_pad,
                                                          const int32_t* __restrict__ cu, const int* __restrict__ tab,
                                                          int B, int Hq) {
    const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows_pad) return;
    const long long bh = row / Npad;
    const int t = static_cast<int>(row - bh * Npad);
    float* acc = dq_acc + row * D;
    for (int c = lane * 4; c < D; c += 128) *reinterpret_cast<float4*>(acc + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    bool valid;
    size_t src, lrow;
    if (!cu) {
        valid = t < N;
        src = (static_cast<size_t>(bh) * N + t) * D;
        lrow = static_cast<size_t>(bh) * N + t;
    } else {
        const int* pad = tab + 2 * B + 1;
        const int sq = last_le(pad, B, t);
        const int tt = t - pad[sq];
        const int len = cu[sq + 1] - cu[sq];
        valid = tab[3 * B + 3] >= 0 && t < pad[B] && tt >= 0 && tt < len;
        const size_t token = static_cast<size_t>(cu[sq]) + tt;
        src = (token * Hq + bh) * D;                 // bh is the head here
        lrow = static_cast<size_t>(bh) * N + token;
    }
    float dsum = 0.f;
    if (valid) {
        for (int c = lane * 2; c < D; c += 64) {
            const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + src + c);
            const uint32_t dv = *reinterpret_cast<const uint32_t*>(dout + src + c);
            dsum += __uint_as_float(ov << 16) * __uint_as_float(dv << 16) +
                    __uint_as_float(ov & 0xFFFF0000u) * __uint_as_float(dv & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (lane == 0) {
        float l2 = INFINITY;
        if (valid) {
            const float l = lse[lrow];
            l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
        }
        lse2[row] = l2;
        Dvec[row] = valid ? dsum : 0.f;
    }
}

// dQ = scale * accumulator -> bf16.  One thread per 4 values of dq (dense
// [B, Hq, N, d]; packed [N, Hq, d]).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ dq_acc, uint16_t* dq, float scale,
                                                        int N, int Npad, long long total4, const int32_t* __restrict__ cu,
                                                        const int* __restrict__ tab, int B, int Hq) {
    const long long e4 = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
    if (e4 >= total4) return;
    const long long e = e4 * 4;
    const long long row = e / D;
    const int c = static_cast<int>(e - row * D);
    size_t arow;
    if (!cu) {
        const long long bh = row / N;              // row of [B*Hq, N]
        const long long t = row - bh * N;
        arow = static_cast<size_t>(bh) * Npad + t;
    } else {
        if (tab[3 * B + 3] < 0) return;            // offsets rejected: dq is left unwritten
        const long long token = row / Hq;          // row of [N, Hq]
        const int h = static_cast<int>(row - token * Hq);
        const int sq = last_le(cu, B, token);
        const int* pad = tab + 2 * B + 1;
        arow = static_cast<size_t>(h) * Npad + pad[sq] + (token - cu[sq]);
    }
    const float4 v = *reinterpret_cast<const float4*>(dq_acc + arow * D + c);
    *reinterpret_cast<uint2*>(dq + e) = make_uint2(pack_bf16x2(v.x * scale, v.y * scale), pack_bf16x2(v.z * scale, v.w * scale));
}

static std::mutex g_bwd_mu;
static bool g_bwd_ready[kMaxDevices];

static int bwd_setup(int dev) {
    std::lock_guard<std::mutex> lock(g_bwd_mu);
    if (g_bwd_ready[dev]) return FA_OK;
    bool good = cudaFuncSetAttribute(fa_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg<64>::kSmemBytes) == cudaSuccess;
    good = good && cudaFuncSetAttribute(fa_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Cfg<128>::kSmemBytes) == cudaSuccess;
    if (!good) return FA_ERR_LAUNCH;
    g_bwd_ready[dev] = true;
    return FA_OK;
}

// Padded rows per head: dense, N rounded up to 128; packed, a bound on the
// sum over sequences of their lengths rounded up to 128.
static size_t padded_rows(int B, int N, bool packed) {
    const size_t n = packed ? static_cast<size_t>(N) + static_cast<size_t>(kBlock) * B : static_cast<size_t>(N);
    return (n + kBlock - 1) / kBlock * kBlock;
}

static size_t workspace_bytes(int B, int Hq, int N, int d, bool packed) {
    const size_t rows = (packed ? 1 : static_cast<size_t>(B)) * Hq * padded_rows(B, N, packed);
    size_t bytes = rows * (d + 2) * sizeof(float);
    if (packed) bytes += (static_cast<size_t>(3) * B + 4) * sizeof(int);
    return bytes;
}

static bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

}  // namespace bwd
}  // namespace fa_sm100

using namespace fa_sm100;

#ifdef FA_TRACE
extern "C" int fa_bwd_trace_set(void* ptr) {
    unsigned long long* q = static_cast<unsigned long long*>(ptr);
    return cudaMemcpyToSymbol(fa_sm100::bwd::g_btrace, &q, sizeof(q)) == cudaSuccess ? 0 : -1;
}
#endif

extern "C" size_t fa_bwd_workspace_bytes(int B, int Hq, int N, int d, int packed) {
    if (B < 0 || Hq < 1 || N < 0 || (d != 64 && d != 128)) return 0;
    if (packed && B > bwd::kMaxSeqsBwd) return 0;
    return bwd::workspace_bytes(B, Hq, N, d, packed != 0);
}

extern "C" int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                      const int32_t* cu_seqlens, void* workspace, size_t workspace_bytes, void* stream) {
    using namespace bwd;
    const bool packed = cu_seqlens != nullptr;
    if (B < 0 || N < 0 || Hq < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (Hkv < 1 || Hq % Hkv != 0) return FA_ERR_GQA;
    if (B == 0 || N == 0) return FA_OK;
    if (packed && B > kMaxSeqsBwd) return FA_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return FA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 16) ||
        (packed && !aligned(cu_seqlens, 4)))
        return FA_ERR_ALIGN;
    const long long npad = (long long)padded_rows(B, N, packed);
    const long long rows_pad = (packed ? 1ll : (long long)B) * Hq * npad;
    if (rows_pad > (1ll << 30) || (long long)B * Hkv * ((N + kBlock - 1) / kBlock) > (1ll << 30) ||
        (long long)Hq * N > (1ll << 30))
        return FA_ERR_SHAPE;
    if (workspace_bytes < bwd::workspace_bytes(B, Hq, N, d, packed)) return FA_ERR_SHAPE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
    DeviceState* ds = nullptr;
    int st = init_device(dev, &ds);
    if (st != FA_OK) return st;
    if ((st = bwd_setup(dev)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    float* dq_acc = static_cast<float*>(workspace);
    float* lse2 = dq_acc + rows_pad * d;
    float* Dvec = lse2 + rows_pad;
    int* tab = packed ? reinterpret_cast<int*>(Dvec + rows_pad) : nullptr;

    Params P;
    std::memset(&P, 0, sizeof(P));
    {
        const uint64_t e = 2;
        bool good;
        if (!packed) {
            const uint32_t box[4] = {64, (uint32_t)kBlock, 1, 1};
            const uint64_t dq_[4] = {(uint64_t)d, (uint64_t)N, (uint64_t)Hq, (uint64_t)B};
            const uint64_t sq[3] = {d * e, (uint64_t)N * d * e, (uint64_t)Hq * N * d * e};
            const uint64_t dk_[4] = {(uint64_t)d, (uint64_t)N, (uint64_t)Hkv, (uint64_t)B};
            const uint64_t sk[3] = {d * e, (uint64_t)N * d * e, (uint64_t)Hkv * N * d * e};
            good = encode_map(&P.tm_q, q, dq_, sq, box) && encode_map(&P.tm_do, dout, dq_, sq, box) &&
                   encode_map(&P.tm_k, k, dk_, sk, box) && encode_map(&P.tm_v, v, dk_, sk, box);
        } else {
            // token-major [N, H, d]: 128 tokens of one head per box
            const uint32_t box[4] = {64, 1, (uint32_t)kBlock, 1};
            const uint64_t dq_[4] = {(uint64_t)d, (uint64_t)Hq, (uint64_t)N, 1};
            const uint64_t sq[3] = {d * e, (uint64_t)Hq * d * e, (uint64_t)N * Hq * d * e};
            const uint64_t dk_[4] = {(uint64_t)d, (uint64_t)Hkv, (uint64_t)N, 1};
            const uint64_t sk[3] = {d * e, (uint64_t)Hkv * d * e, (uint64_t)N * Hkv * d * e};
            good = encode_map(&P.tm_q, q, dq_, sq, box) && encode_map(&P.tm_do, dout, dq_, sq, box) &&
                   encode_map(&P.tm_k, k, dk_, sk, box) && encode_map(&P.tm_v, v, dk_, sk, box);
        }
        if (!good) return FA_ERR_LAUNCH;
    }
    P.lse2 = lse2;
    P.Dvec = Dvec;
    P.dq_acc = dq_acc;
    P.cu = cu_seqlens;
    P.tab = tab;
    P.dk = static_cast<uint16_t*>(dk);
    P.dv = static_cast<uint16_t*>(dv);
    P.status = ds->status;
    P.B = B;
    P.Hq = Hq;
    P.Hkv = Hkv;
    P.N = N;
    P.Npad = (int)npad;
    P.group = Hq / Hkv;
    P.causal = causal ? 1 : 0;
    P.packed = packed ? 1 : 0;
    P.scale = scale;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.timeout_ns = 2000000000ull;

    if (packed) fa_bwd_tables_kernel<<<1, 1024, 0, s>>>(cu_seqlens, B, N, Hkv, tab, ds->status);
    const unsigned prep_grid = static_cast<unsigned>((rows_pad + 7) / 8);
    // dense: the exact number of work units; packed: one CTA per SM (the count is on the device)
    const long long units = packed ? (long long)ds->num_sms
                                   : (long long)B * Hkv * (((N + kBlock - 1) / kBlock + 1) / 2);
    const int grid = (int)std::min<long long>(units, ds->num_sms);
    const long long total4 = (packed ? (long long)N * Hq : (long long)B * Hq * N) * d / 4;
    const unsigned post_grid = static_cast<unsigned>((total4 + 255) / 256);
    const uint16_t* o16 = static_cast<const uint16_t*>(o);
    const uint16_t* do16 = static_cast<const uint16_t*>(dout);
    if (d == 64) {
        fa_bwd_prep_kernel<64><<<prep_grid, 256, 0, s>>>(o16, do16, lse, lse2, Dvec, dq_acc, N, (int)npad, rows_pad,
                                                          cu_seqlens, tab, B, Hq);
        fa_bwd_kernel<64><<<grid, kThreads, Cfg<64>::kSmemBytes, s>>>(P);
        fa_bwd_dq_kernel<64><<<post_grid, 256, 0, s>>>(dq_acc, static_cast<uint16_t*>(dq), scale, N, (int)npad, total4,
                                                        cu_seqlens, tab, B, Hq);
    } else {
        fa_bwd_prep_kernel<128><<<prep_grid, 256, 0, s>>>(o16, do16, lse, lse2, Dvec, dq_acc, N, (int)npad, rows_pad,
                                                           cu_seqlens, tab, B, Hq);
        fa_bwd_kernel<128><<<grid, kThreads, Cfg<128>::kSmemBytes, s>>>(P);
        fa_bwd_dq_kernel<128><<<post_grid, 256, 0, s>>>(dq_acc, static_cast<uint16_t*>(dq), scale, N, (int)npad,
                                                         total4, cu_seqlens, tab, B, Hq);
    }
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}
