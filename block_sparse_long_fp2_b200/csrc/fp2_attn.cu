// Stage 2 of FlashPrefill V2 (Figure 3 / Figure 4 of the metallab.ai summary
// of arXiv 2608.19758): sparse attention over the selected key blocks with
// the mean correction merged into the same online softmax.
//
// One persistent CTA per SM (320 threads) takes work items from the schedule
// the plan wrote (longest rows first within L2-sized chunks of kv-heads).  A
// work item is one CSR row (sequence s, kv-head g, query block i), or one
// count-balanced split of a long row's tiles (Table 7), restricted to two
// PackGQA query tiles of 128 rows each (the G heads x B tokens of the row,
// packed head-major).  Both tiles share every K/V tile the CTA streams, so
// K/V cross HBM once per kv-head (PackGQA).  A split writes its normalised
// O and log-sum-exp to scratch; k_combine merges a row's splits.  For
// chunked prefill (CHUNK) the queries of sequence s are the positions from
// its chunk offset on, read from and written to the chunk's own tokens.
//
// Roles (warp specialisation):
//   warps 0-3   softmax warpgroup of query tile 0 (TMEM lanes 0-127)
//   warps 4-7   softmax warpgroup of query tile 1
//   warp 8      TMA producer: Q tiles, then per kept block its K and V tiles
//               (through the page table when paged), then per pseudo tile
//               up to B block means Kbar/Vbar (bf16; e4m3 with the key means
//               in two terms, hi and lo, in two ring slots); a ring of K-or-V
//               slots (as many as shared memory holds, 5 at d = B = 128).
//   warp 9      allocates tensor memory and issues every tcgen05 MMA:
//               S_m = Q_m K^T into TMEM, O_m += P_m V with P_m read from TMEM
//               (P overwrites its own S columns).  Issue order for K/V tile n:
//               S0(n), P1(n-1).V, S1(n), P0(n).V.  Every commit that publishes
//               S_m(n) therefore also covers P_m(n-1).V, so the softmax warps
//               may rescale O_m and overwrite the P_m columns as soon as S_m(n)
//               is visible; and S_m(n+1) is issued only after the issuer saw
//               P_m(n) published, i.e. after the softmax finished reading S_m(n).
//
// Mean correction (Figure 4): each skipped, fully visible block j adds one
// pseudo-key with key Kbar_j, value Vbar_j and logit bias ln n_j = ln B.
// Up to B skipped blocks form one pseudo tile, run through exactly the same
// MMA + softmax path as a real K/V tile, with the columns of kept blocks
// (and of blocks j >= i) masked out.  In e4m3 the pseudo logits are
// Q (Kbar_hi + Kbar_lo)^T, two MMAs into the same accumulator, so the key
// means enter with about 2^-8 relative error rather than e4m3's 2^-4.
//
// Every wait is bounded (about a second); a timeout records
// FP2_STATUS_TIMEOUT, all roles stop, in-flight copies and MMAs are drained
// and the tensor memory is released before the CTA exits.
#include <cfloat>
#include <cmath>

#include "fp2_device.cuh"

namespace fp2 {

namespace {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;     // issues every MMA; owns the tensor memory
// Ring slots for K / V tiles: as many as fit beside the two query tiles in
// the 227 KiB of shared memory a CTA may use (at most 8).
constexpr int kMaxSmem = 232448;
constexpr int kMaxSlots = 8;
template <int HD, int BLK, bool F8>
constexpr int ring_slots() {
    const int elt = F8 ? 1 : 2;
    const int avail = (kMaxSmem - 512 - 1024 - 2 * kTileM * HD * elt) / (BLK * HD * elt);
    return avail < kMaxSlots ? avail : kMaxSlots;
}

constexpr int pow2_ceil(int x) {
    int p = 32;
    while (p < x) p <<= 1;
    return p;
}

// F8: e4m3 Q/K/V (kind::f8f6f4 MMAs, K = 32 per instruction); otherwise bf16
// (kind::f16, K = 16).  Operand rows are stored as 128-byte swizzle atoms.
template <int HD, int BLK, bool F8>
struct Cfg {
    static constexpr int kElt = F8 ? 1 : 2;              // bytes per element
    static constexpr int kRowBytes = HD * kElt;          // one row of Q / K / V
    static constexpr int kAtoms = kRowBytes / 128;       // 128-byte atoms per row
    static constexpr int kAtomElems = 128 / kElt;        // elements per atom row
    static constexpr int kKStep = F8 ? 32 : 16;          // K elements per MMA instruction
    static_assert(kAtoms >= 1, "rows must span whole 128-byte atoms");
    static constexpr int kSlots = ring_slots<HD, BLK, F8>();
    static constexpr int kQBytes = kTileM * kRowBytes;   // one 128-row query tile
    static constexpr int kSlotBytes = BLK * kRowBytes;   // one K or V tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffSlot = 2 * kQBytes;
    static constexpr int kOffBar = kOffSlot + kSlots * kSlotBytes;
    static_assert(kSlots >= 3, "the K/V ring needs at least three slots");
    static constexpr int kSmemBytes = kOffBar + 512 + 1024;   // barriers + alignment slack
    static_assert(kSmemBytes <= kMaxSmem, "shared memory budget");
    static constexpr int kColS0 = 0;
    static constexpr int kColS1 = BLK;
    static constexpr int kColO0 = 2 * BLK;
    static constexpr int kColO1 = 2 * BLK + HD;
    static constexpr int kTmemCols = pow2_ceil(2 * (BLK + HD));
    static constexpr int kAtomQ = kTileM * 128;          // bytes between column atoms of Q
    static constexpr int kAtomKV = BLK * 128;            // bytes between column atoms of K / V
    // Each MMA covers kKStep elements = 32 bytes of a row, four per atom;
    // P is packed 32 bits per TMEM column, so one K-step of P.V is 8 columns.
    static constexpr uint32_t kIdescS =
        F8 ? idesc_e4m3(kTileM, BLK, false) : idesc_bf16(kTileM, BLK, false);
    static constexpr uint32_t kIdescO =
        F8 ? idesc_e4m3(kTileM, HD, true) : idesc_bf16(kTileM, HD, true);
    // P <= 2^headroom: bf16 P and fp32 sums allow 2^64; e4m3 P' = P s_V K_row
    // must stay <= 448, which K_row = 448 / (2^8 max s_V) ensures for 2^8.
    static constexpr float kHeadroom = F8 ? 8.0f : 64.0f;
};

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[kMaxSlots], kv_empty[kMaxSlots];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_full[2], o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct AttnParams {
    Dims D;
    const int32_t* cu_seqlens;
    const int32_t* page_table;
    const int32_t* row_ptr;
    const int32_t* col_idx;
    const uint32_t* kept_mask;
    const int32_t* block_seq;
    const int32_t* cu_blocks;
    const int32_t* meta_valid;
    int32_t* status;
    uint16_t* o;
    float* lse;
    // FP8 only: per-(block, head) scales of Q, K, V; per-chunk scales of the
    // e4m3 block means; largest V scale per (sequence, kv-head)
    const float* q_scale;
    const float* k_scale;
    const float* v_scale;
    const float* kbar_scale;
    const float* vbar_scale;
    const float* vmax;
    uint32_t flags;
    int n_mtiles;   // 128-row query tiles per row = G * B / 128
    // work schedule (built with the plan) and the scratch of split rows
    const int4* sched;
    float* split_o;
    float* split_lse;
    const int32_t* slot_item;
    // queries: q, o and lse hold Tq tokens; sequence s's queries start at
    // token cu_q[s] and position q_off[s] (a chunk; cu_seqlens and 0 otherwise)
    const int32_t* cu_q;
    const int32_t* q_off;
    int64_t Tq;
    int64_t n_items;   // work items in the schedule
    int64_t n_slots;   // n_items rounded up to whole passes of the grid
    int64_t n_split_rows;   // rows of the split scratch (slots x G x B)
    bool zigzag;       // odd passes run backwards
};

// One work item: split k of S of row (s, g, i), query tiles 2*mp, 2*mp+1.
struct Item {
    int s, g, i, mp;
    int k, S, slot;      // split, splits of the row, first split slot of the row
    int64_t b, r;
    int kbeg, kend;      // CSR range of the row
    int tok0, L;         // first token of the sequence, its length
    int b0;              // first global block of the sequence
    bool has_m1;
    bool ok;             // false: the debug build's checks rejected the entry
};

// The schedule lists the items longest row first (within a chunk of kv-heads
// whose K/V share L2).  CTA c takes the c-th item of every pass over the grid;
// with few passes (zigzag) it takes the c-th from the end on odd passes,
// which evens out the rows' decreasing lengths across the CTAs (measured
// 6-7 % faster at 8K-16K tokens per layer, 2 % slower at 128K, where the
// passes are many and the lengths wrap around every kv-head).  Returns
// n_items or more for a slot without an item.
__device__ __forceinline__ int64_t sched_index(int64_t w, bool zigzag) {
    const int64_t pass = w / gridDim.x;
    return (zigzag && (pass & 1)) ? pass * gridDim.x + (gridDim.x - 1 - blockIdx.x) : w;
}

__device__ __forceinline__ Item decode_item(const AttnParams& P, int64_t w) {
    Item it;
    const int4 e = __ldg(P.sched + w);
    it.b = e.x;
    it.g = e.y & 0xFFFF;
    it.mp = e.y >> 16;
    it.k = e.z & 0xFFFF;
    it.S = e.z >> 16;
    it.slot = e.w;
    it.ok = FP2_CHECK(it.b >= 0 && it.b < P.D.NB && it.g < P.D.Hkv && 2 * it.mp < P.n_mtiles &&
                          it.S >= 1 && it.S <= kMaxSplits && it.k < it.S,
                      P.status);
    if (!it.ok) it.b = 0;
    it.s = P.block_seq[it.b];
    it.b0 = P.cu_blocks[it.s];
    it.i = (int)(it.b - it.b0);
    it.r = (int64_t)it.g * P.D.NB + it.b;
    it.kbeg = P.row_ptr[it.r];
    it.kend = P.row_ptr[it.r + 1];
    it.ok = it.ok && FP2_CHECK(it.kbeg >= 0 && it.kbeg <= it.kend && it.kend <= P.D.nnz_cap &&
                                   it.kend - it.kbeg <= it.i + 1,
                               P.status);
    if (!it.ok) it.kend = it.kbeg;
    it.tok0 = P.cu_seqlens[it.s];
    it.L = P.cu_seqlens[it.s + 1] - it.tok0;
    it.has_m1 = 2 * it.mp + 1 < P.n_mtiles;
    return it;
}

enum TileKind { kFull = 0, kDiag = 1, kPseudo = 2 };

// Walks the tiles of an item: the kept blocks in CSR order, then the pseudo
// tiles that contain at least one skipped block.  Every role runs the same
// walk, so they agree on the sequence without exchanging it.  The next
// column id is loaded one step ahead and the non-empty pseudo tiles are
// found once per item, so advancing never waits on a global load.
template <int BLK>
struct TileWalk {
    static constexpr int W = BLK / 32;
    const int32_t* cols;
    const uint32_t* mask;
    int n_kept, t, i, pt, n_pt;
    int j_next;          // col_idx[t] (valid when t < n_kept)
    uint32_t pt_bits;    // bit p set: pseudo tile p (p < 32) holds a skipped block
    int32_t* status;

    __device__ __forceinline__ void init(const AttnParams& P, const Item& it) {
        status = P.status;
        cols = P.col_idx + it.kbeg;
        n_kept = it.kend - it.kbeg;
        t = 0;
        i = it.i;
        mask = P.kept_mask + it.r * P.D.mask_words;
        pt = 0;
        n_pt = (P.flags & FP2_NO_CORRECTION) ? 0 : (it.i + BLK - 1) / BLK;
        pt_bits = 0;
        const int n_small = n_pt < 32 ? n_pt : 32;
        for (int p = 0; p < n_small; ++p) pt_bits |= has_skip(p) ? (1u << p) : 0u;
        if (it.S > 1) {
            // count-balanced split: tiles [k n / S, (k + 1) n / S) of the n tiles
            // of the row; the walk's ends are moved onto that range
            const int n = count();
            const int t0 = (int)((int64_t)it.k * n / it.S);
            const int t1 = (int)((int64_t)(it.k + 1) * n / it.S);
            if (t1 <= n_kept) {
                n_kept = t1;
                n_pt = 0;
            } else {
                int p = 0;
                for (int r = t1 - n_kept; r > 0 && p < n_pt; ++p) r -= pt_nonempty(p) ? 1 : 0;
                n_pt = p;
            }
            if (t0 <= n_kept) {
                t = t0;
            } else {
                t = n_kept;
                for (int r = t0 - n_kept; r > 0 && pt < n_pt; ++pt) r -= pt_nonempty(pt) ? 1 : 0;
            }
        }
        j_next = t < n_kept ? __ldg(cols + t) : 0;
    }
    // skip bits of blocks BLK*pt + 32*w .. +31 (skipped = visible, j < i, not kept)
    __device__ __forceinline__ uint32_t skip_word(int p, int w) const {
        const int j0 = BLK * p + 32 * w;
        if (j0 >= i) return 0u;
        const uint32_t valid = (j0 + 32 <= i) ? 0xFFFFFFFFu : ((1u << (i - j0)) - 1u);
        return ~__ldg(mask + j0 / 32) & valid;
    }
    __device__ __forceinline__ bool has_skip(int p) const {
        uint32_t any = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) any |= skip_word(p, w);
        return any != 0;
    }
    __device__ __forceinline__ bool pt_nonempty(int p) const {
        return p < 32 ? ((pt_bits >> p) & 1u) != 0 : has_skip(p);
    }
    // Advances to the next tile; returns false at the end.
    __device__ __forceinline__ bool next(int& kind, int& j) {
        if (t < n_kept) {
            j = j_next;
            if (!FP2_CHECK(j >= 0 && j <= i, status)) j = i;   // a column outside the row
            ++t;
            if (t < n_kept) j_next = __ldg(cols + t);
            kind = (j == i) ? kDiag : kFull;
            return true;
        }
        while (pt < n_pt && !pt_nonempty(pt)) ++pt;
        if (pt >= n_pt) return false;
        j = pt++;
        kind = kPseudo;
        return true;
    }
    // Tiles left in the walk (kept blocks + non-empty pseudo tiles), so a role
    // that needs no column ids can count tiles without loading them.
    __device__ __forceinline__ int count() const {
        int n = n_kept - t;
        const int hi = n_pt < 32 ? n_pt : 32;
        if (pt < hi) {
            const uint32_t below_hi = hi == 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u);
            n += __popc(pt_bits & below_hi & ~((1u << pt) - 1u));
        }
        for (int p = pt > 32 ? pt : 32; p < n_pt; ++p) n += has_skip(p) ? 1 : 0;
        return n;
    }
};

// Whether split k of S of a row with n tiles has any tile.
__device__ __forceinline__ bool split_nonempty(int k, int S, int n) {
    return (int64_t)(k + 1) * n / S > (int64_t)k * n / S;
}

// Uniform wait for a whole warp: every lane waits, then all agree.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars& B, int32_t* status) {
    bool ok = mbar_wait(bar, parity, &B.abort, status);
    return __all_sync(0xffffffffu, ok);
}

// Columns 32*c .. 32*c+31 of a tile that take part in the softmax: all of a
// full block, the causal part (column <= tok) of the diagonal block, and the
// skipped blocks of a pseudo tile.
template <int BLK>
__device__ __forceinline__ uint32_t col_bits(int kind, int tok, const TileWalk<BLK>& walk, int j,
                                             int c) {
    if (kind == kFull) return 0xFFFFFFFFu;
    if (kind == kDiag) {
        const int lim = tok - 32 * c;
        return lim >= 31 ? 0xFFFFFFFFu : (lim < 0 ? 0u : ((2u << lim) - 1u));
    }
    return walk.skip_word(j, c);
}

// ---------------------------------------------------------------------------
// producer (warp 8, one lane)
// ---------------------------------------------------------------------------

template <int HD, int BLK, bool F8, bool CHUNK>
__device__ void producer(const AttnParams& P, Bars& B, uint8_t* smem, const CUtensorMap* tm_q,
                         const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_kbar, const CUtensorMap* tm_vbar,
                         const CUtensorMap* tm_kbar_lo) {
    using C = Cfg<HD, BLK, F8>;
    const Dims& D = P.D;
    uint32_t qcnt[2] = {0, 0}, qloaded[2] = {0, 0};
    uint32_t ld = 0;                 // K/V loads issued (slot = ld % kSlots)
    constexpr int kSlots = C::kSlots;
    uint32_t issued[kMaxSlots] = {0, 0, 0, 0, 0, 0, 0, 0};
    const bool paged = D.page_size != 0;
    for (int64_t w = blockIdx.x; w < P.n_slots; w += gridDim.x) {
        const int64_t o = sched_index(w, P.zigzag);
        if (o >= P.n_items) continue;
        const Item it = decode_item(P, o);
        if (!it.ok) continue;
        TileWalk<BLK> walk;
        walk.init(P, it);
        if (walk.count() == 0) continue;   // a split without tiles
        // q token of position 0 of the sequence (for a chunk that starts inside
        // the block, rows before the chunk read zeros or another sequence's
        // queries: they are never written)
        const int qtok = CHUNK ? P.cu_q[it.s] - P.q_off[it.s] : it.tok0;
        for (int m = 0; m < 2; ++m) {
            if (m == 1 && !it.has_m1) break;
            if (!mbar_wait(&B.q_empty[m], (qcnt[m] & 1) ^ 1, &B.abort, P.status)) goto drain;
            ++qcnt[m];
            if (P.flags & FP2_DEBUG_DROP_Q_LOAD) continue;   // fault injection: never arrives
            qloaded[m] = qcnt[m];
            mbar_arrive_expect_tx(&B.q_full[m], C::kQBytes);
            uint8_t* qdst = smem + C::kOffQ + m * C::kQBytes;
            const int mt = 2 * it.mp + m;
#pragma unroll
            for (int ht = 0; ht < kTileM / BLK; ++ht) {
                const int hl = (kTileM * mt) / BLK + ht;
#pragma unroll
                for (int a = 0; a < C::kAtoms; ++a)
                    tma_load_3d(qdst + a * C::kAtomQ + ht * BLK * 128, tm_q, &B.q_full[m],
                                C::kAtomElems * a, it.g * D.G + hl, qtok + it.i * BLK);
            }
        }
        int kind, j;
        while (walk.next(kind, j)) {
            // ring entries of the tile: K and V; an e4m3 pseudo tile's keys
            // take two (the two e4m3 terms of the key means)
            const int n_ent = (F8 && kind == kPseudo) ? 3 : 2;
            for (int e = 0; e < n_ent; ++e) {
                const int kv = e == n_ent - 1 ? 1 : 0;
                const int slot = ld % kSlots;
                const uint32_t use = ld / kSlots;
                if (!mbar_wait(&B.kv_empty[slot], (use & 1) ^ 1, &B.abort, P.status)) goto drain;
                ++ld;
                issued[slot] = use + 1;
                uint64_t* bar = &B.kv_full[slot];
                mbar_arrive_expect_tx(bar, C::kSlotBytes);
                uint8_t* dst = smem + C::kOffSlot + slot * C::kSlotBytes;
                if (kind == kPseudo) {
                    FP2_CHECK(it.b0 + j * BLK < D.NB, P.status);   // (beyond: zero fill)
                    const CUtensorMap* tm = kv == 1 ? tm_vbar : (e == 0 ? tm_kbar : tm_kbar_lo);
#pragma unroll
                    for (int a = 0; a < C::kAtoms; ++a)
                        tma_load_3d(dst + a * C::kAtomKV, tm, bar, C::kAtomElems * a, it.g,
                                    it.b0 + j * BLK);
                } else if (!paged) {
                    const CUtensorMap* tm = kv == 0 ? tm_k : tm_v;
#pragma unroll
                    for (int a = 0; a < C::kAtoms; ++a)
                        tma_load_3d(dst + a * C::kAtomKV, tm, bar, C::kAtomElems * a, it.g,
                                    it.tok0 + j * BLK);
                } else {
                    const CUtensorMap* tm = kv == 0 ? tm_k : tm_v;
                    const int n_pages_s = (it.L + 63) / 64;
#pragma unroll
                    for (int pg = 0; pg < BLK / 64; ++pg) {
                        const int pi = (j * BLK) / 64 + pg;
                        int id = D.num_pages;   // out of range: the copy fills zeros
                        if (pi < n_pages_s && FP2_CHECK(pi < D.pt_stride, P.status)) {
                            const int e = P.page_table[(int64_t)it.s * D.pt_stride + pi];
                            if (e >= 0 && e < D.num_pages) id = e;
                            else atomicOr(P.status, (int32_t)FP2_STATUS_BAD_PAGE);
                        }
#pragma unroll
                        for (int a = 0; a < C::kAtoms; ++a)
                            tma_load_4d(dst + a * C::kAtomKV + pg * 64 * 128, tm, bar,
                                        C::kAtomElems * a, it.g, 0, id);
                    }
                }
            }
        }
    }
drain:
    // Let every copy this thread started land before the CTA may exit.
    for (int s = 0; s < kSlots; ++s)
        if (issued[s]) mbar_wait_drain(&B.kv_full[s], (issued[s] - 1) & 1, P.status);
    if (!(P.flags & FP2_DEBUG_DROP_Q_LOAD))
        for (int m = 0; m < 2; ++m)
            if (qloaded[m]) mbar_wait_drain(&B.q_full[m], (qloaded[m] - 1) & 1, P.status);
}

// ---------------------------------------------------------------------------
// MMA issuer (warp 9, one lane)
// ---------------------------------------------------------------------------

// The shared-memory descriptors of one operand tile differ between K-steps
// only in the start-address field (bits 0-13, address / 16); the tiles never
// cross 256 KiB, so the field never carries and a K-step is one add of a
// compile-time constant to a descriptor built once per kernel.
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
    return d + static_cast<uint64_t>(bytes >> 4);
}

// S = Q K^T (accumulate: S += Q K^T, for the second term of e4m3 key means).
template <int HD, int BLK, bool F8>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint64_t q_desc, uint64_t k_desc,
                                        bool accumulate = false) {
    using C = Cfg<HD, BLK, F8>;
#pragma unroll
    for (int kk = 0; kk < HD / C::kKStep; ++kk) {
        const uint64_t a = desc_add(q_desc, (kk / 4) * C::kAtomQ + (kk % 4) * 32);
        const uint64_t b = desc_add(k_desc, (kk / 4) * C::kAtomKV + (kk % 4) * 32);
        const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
        if (F8) umma_f8(tmem_s, a, b, C::kIdescS, acc);
        else umma_f16(tmem_s, a, b, C::kIdescS, acc);
    }
}

template <int HD, int BLK, bool F8>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t v_desc,
                                         bool accumulate) {
    using C = Cfg<HD, BLK, F8>;
#pragma unroll
    for (int kk = 0; kk < BLK / C::kKStep; ++kk) {
        const uint64_t b = desc_add(v_desc, kk * C::kKStep * 128);
        const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
        if (F8) umma_f8_ts(tmem_o, tmem_p + kk * 8, b, C::kIdescO, acc);
        else umma_f16_ts(tmem_o, tmem_p + kk * 8, b, C::kIdescO, acc);
    }
}

struct PrevTile {
    bool valid, has_m1, first, last;
    int vslot;
};

// Position in the K/V ring: slot and how many times it has been used before.
struct RingPos {
    int slot;
    uint32_t use;
};
template <int kSlots>
__device__ __forceinline__ RingPos ring_take(RingPos& next) {
    const RingPos cur = next;
    if (++next.slot == kSlots) {
        next.slot = 0;
        ++next.use;
    }
    return cur;
}

// The MMA issuer (one lane of warp kMmaWarp).  A tcgen05.mma costs its
// issuing thread ~50 cycles, about its 64-cycle execution time, so a single
// thread issues every MMA in the order S0(n), P1(n-1).V, S1(n), P0(n).V
// that keeps the two query tiles' chains interleaved.  The loop is rotated
// so that S0(n+1) follows P0(n).V directly (the next tile's K is usually long
// resident): the loop overhead and the wait for P1 fall on the other query
// tile's chain, which is half a period behind.
template <int HD, int BLK, bool F8>
__device__ void mma_issuer(const AttnParams& P, Bars& B, uint8_t* smem) {
    using C = Cfg<HD, BLK, F8>;
    constexpr int kSlots = C::kSlots;
    const uint32_t tb = B.tmem_base;
    const uint32_t s_base = smem_u32(smem);
    const uint64_t q_desc[2] = {smem_desc_sw128(s_base + C::kOffQ, 16, 1024),
                                smem_desc_sw128(s_base + C::kOffQ + C::kQBytes, 16, 1024)};
    // descriptors of ring slot 0 as a K (K-major) and as a V (MN-major) operand
    const uint64_t k_desc0 = smem_desc_sw128(s_base + C::kOffSlot, 16, 1024);
    const uint64_t v_desc0 = smem_desc_sw128(s_base + C::kOffSlot, C::kAtomKV, 1024);
    const uint32_t t_s[2] = {tb + C::kColS0, tb + C::kColS1};
    const uint32_t t_o[2] = {tb + C::kColO0, tb + C::kColO1};
    uint32_t qcnt[2] = {0, 0}, pcnt[2] = {0, 0}, ocnt[2] = {0, 0};
    RingPos ring{0, 0};
    PrevTile prev{false, false, false, false, 0};

    auto pv1 = [&](const PrevTile& pt) -> bool {
        if (!mbar_wait(&B.p_full[1], pcnt[1] & 1, &B.abort, P.status)) return false;
        ++pcnt[1];
        if (pt.first && !mbar_wait(&B.o_free[1], (ocnt[1] & 1) ^ 1, &B.abort, P.status)) return false;
        tc_fence_after();
        issue_pv<HD, BLK, F8>(t_o[1], t_s[1], desc_add(v_desc0, pt.vslot * C::kSlotBytes), !pt.first);
        umma_commit(&B.kv_empty[pt.vslot]);
        if (pt.last) {
            umma_commit(&B.o_full[1]);
            ++ocnt[1];
        }
        return true;
    };
    // The K ring entries of one tile: its K tile, and for an e4m3 pseudo tile
    // the second term of the key means in the next entry (lo).
    struct KPos {
        RingPos k, lo;
        bool two;
    };
    auto kdesc = [&](const RingPos& r) { return desc_add(k_desc0, r.slot * C::kSlotBytes); };
    // S_m = Q_m K^T of the tile's K entries (waits for them to land)
    auto issue_sm = [&](int m, const KPos& kk) -> bool {
        if (!mbar_wait(&B.kv_full[kk.k.slot], kk.k.use & 1, &B.abort, P.status)) return false;
        if (kk.two && !mbar_wait(&B.kv_full[kk.lo.slot], kk.lo.use & 1, &B.abort, P.status))
            return false;
        tc_fence_after();
        issue_s<HD, BLK, F8>(t_s[m], q_desc[m], kdesc(kk.k));
        if (kk.two) issue_s<HD, BLK, F8>(t_s[m], q_desc[m], kdesc(kk.lo), true);
        return true;
    };
    auto release_k = [&](const KPos& kk) {
        umma_commit(&B.kv_empty[kk.k.slot]);
        if (kk.two) umma_commit(&B.kv_empty[kk.lo.slot]);
    };
    // S0 = Q0 K^T
    auto s0 = [&](const KPos& kk, bool has_m1, bool last) -> bool {
        if (!issue_sm(0, kk)) return false;
        umma_commit(&B.s_full[0]);
        if (!has_m1) {
            release_k(kk);
            if (last) umma_commit(&B.q_empty[0]);
        }
        return true;
    };

    for (int64_t w = blockIdx.x; w < P.n_slots; w += gridDim.x) {
        const int64_t o = sched_index(w, P.zigzag);
        if (o >= P.n_items) continue;
        const Item it = decode_item(P, o);
        if (!it.ok) continue;
        // The issuer needs no column ids, only the tile count (and, for e4m3,
        // where the pseudo tiles start): its loop issues no global loads,
        // which would otherwise hold up its barrier probes.
        int n_tiles, n_real;
        {
            TileWalk<BLK> walk;
            walk.init(P, it);
            n_tiles = walk.count();
            n_real = walk.n_kept - walk.t;   // tiles before the pseudo tiles
        }
        if (n_tiles == 0) continue;
        auto take_tile = [&](int n, KPos& kk, RingPos& v) {
            kk.k = ring_take<kSlots>(ring);
            kk.two = F8 && n >= n_real;
            if (kk.two) kk.lo = ring_take<kSlots>(ring);
            v = ring_take<kSlots>(ring);
        };
        KPos kp;
        RingPos vp;
        take_tile(0, kp, vp);
        if (!mbar_wait(&B.q_full[0], qcnt[0] & 1, &B.abort, P.status)) goto drain;
        ++qcnt[0];
        if (!s0(kp, it.has_m1, n_tiles == 1)) goto drain;
        for (int n = 0; n < n_tiles; ++n) {
            const bool first = n == 0;
            const bool last = n == n_tiles - 1;
            // P1.V of the previous tile
            if (prev.valid && prev.has_m1) {
                if (!pv1(prev)) goto drain;
            }
            // S1 = Q1 K^T
            if (it.has_m1) {
                if (first) {
                    if (!mbar_wait(&B.q_full[1], qcnt[1] & 1, &B.abort, P.status)) goto drain;
                    ++qcnt[1];
                }
                if (!issue_sm(1, kp)) goto drain;
                umma_commit(&B.s_full[1]);
                release_k(kp);
                if (last) {
                    umma_commit(&B.q_empty[0]);
                    umma_commit(&B.q_empty[1]);
                }
            }
            // P0.V of this tile
            if (!mbar_wait(&B.kv_full[vp.slot], vp.use & 1, &B.abort, P.status)) goto drain;
            if (!mbar_wait(&B.p_full[0], pcnt[0] & 1, &B.abort, P.status)) goto drain;
            ++pcnt[0];
            if (first && !mbar_wait(&B.o_free[0], (ocnt[0] & 1) ^ 1, &B.abort, P.status)) goto drain;
            tc_fence_after();
            issue_pv<HD, BLK, F8>(t_o[0], t_s[0], desc_add(v_desc0, vp.slot * C::kSlotBytes), !first);
            if (!it.has_m1) umma_commit(&B.kv_empty[vp.slot]);
            if (last) {
                umma_commit(&B.o_full[0]);
                ++ocnt[0];
            }
            prev = PrevTile{true, it.has_m1, first, last, vp.slot};
            // S0 of the next tile right away
            if (!last) {
                take_tile(n + 1, kp, vp);
                if (!s0(kp, it.has_m1, n + 1 == n_tiles - 1)) goto drain;
            }
        }
    }
    if (prev.valid && prev.has_m1) pv1(prev);
drain:
    // Wait until every MMA issued above has completed.
    umma_commit(&B.drain);
    mbar_wait_drain(&B.drain, 0, P.status);
}

template <int BLK, bool MASKED>
__device__ __forceinline__ uint32_t chunk_bits(int kind, int tok, const TileWalk<BLK>& walk, int j,
                                               int c32) {
    return MASKED ? col_bits(kind, tok, walk, j, c32) : 0xFFFFFFFFu;
}

// 32 columns of P = 2^(s * scale + shift), written into tensor memory over
// the first part of the 32 S columns just read: the A operand of the P.V MMA.
//   bf16: 16 packed pairs (keys 2c, 2c+1 in column c), columns [t_p, t_p+16).
//   e4m3: P' = P * pfac packed four per column, columns [t_p, t_p+8), pfac
//   entering through the shift (as log2 pfac).
// The fp32 row sum accumulates the P written (P' for e4m3).
// Exponentials computed on the FMA pipe (exp2_fma2) instead of MUFU ex2: the
// pairs p of a 32-column chunk with p % 8 < kEmuPairs / 2, i.e. kEmuPairs of
// the 16 pairs (both units then share the softmax's exponentials).
#ifndef FP2_EXP2_FMA_PAIRS_BF16
#define FP2_EXP2_FMA_PAIRS_BF16 0
#endif
#ifndef FP2_EXP2_FMA_PAIRS_E4M3
#define FP2_EXP2_FMA_PAIRS_E4M3 0
#endif
template <bool F8>
constexpr int emu_pairs() { return F8 ? FP2_EXP2_FMA_PAIRS_E4M3 : FP2_EXP2_FMA_PAIRS_BF16; }

template <bool MASKED, bool F8>
__device__ __forceinline__ void p32(const uint32_t (&r)[32], uint32_t vb, uint32_t t_p,
                                    uint64_t scale2, uint64_t shift2, uint64_t& sum2) {
    constexpr int kEmu = emu_pairs<F8>();
    float p[32];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float s0 = __uint_as_float(r[e]), s1 = __uint_as_float(r[e + 1]);
        if (MASKED) {
            s0 = ((vb >> e) & 1u) ? s0 : -INFINITY;
            s1 = ((vb >> (e + 1)) & 1u) ? s1 : -INFINITY;
        }
        const uint64_t x2 = f2_fma(f2_pack(s0, s1), scale2, shift2);
        if ((e / 2) % 8 < kEmu / 2) {
            f2_unpack(exp2_fma2(x2), p[e], p[e + 1]);
        } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p[e] = ex2_approx(x0);
            p[e + 1] = ex2_approx(x1);
        }
        sum2 = f2_add(sum2, f2_pack(p[e], p[e + 1]));
    }
    if (F8) {
        uint32_t packed[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            packed[q] = pack_e4m3x4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
        tmem_st8(t_p, packed);
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t packed[8];
#pragma unroll
            for (int e2 = 0; e2 < 8; ++e2) packed[e2] = pack_bf16x2(p[16 * h + 2 * e2], p[16 * h + 2 * e2 + 1]);
            tmem_st8(t_p + 8 * h, packed);
        }
    }
}

template <bool MASKED>
__device__ __forceinline__ float max32(const uint32_t (&r)[32], uint32_t vb) {
    float mx = -INFINITY;
    if (MASKED) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if ((vb >> e) & 1u) mx = fmaxf(mx, __uint_as_float(r[e]));
    } else {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
            m0 = fmax3(m0, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
            m1 = fmax3(m1, __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
            m2 = fmax3(m2, __uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]));
            m3 = fmax3(m3, __uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
        }
        mx = fmaxf(fmax3(m0, m1, m2), m3);
    }
    return mx;
}

// Softmax state of one query row (one thread): the running reference
// maximum (log2 units), the fp32 row sum, the row's O accumulator columns.
struct RowState {
    float m_ref, l;
    uint32_t t_o;
    bool o_valid;   // O holds data (false before the first P.V of the row)
};

// Moves the reference maximum of this thread's row to m_new (>= m_ref):
// O, l, the partial sum of the current tile and the P columns already
// written for it (cols [t_p0, t_p0 + n_pcols)) are scaled by 2^(m_ref - m_new).
// Warp-collective (tensor memory accesses); lanes whose reference does not
// move use the factor 1.
template <int HD, bool F8>
__device__ __forceinline__ void move_reference(RowState& st, float m_new, uint64_t& sum2, uint32_t t_p0,
                                               int n_pcols) {
    tmem_st_wait();   // the P columns read back below were stored by this thread
    const float alpha = m_new > st.m_ref ? ex2_approx(st.m_ref - m_new) : 1.0f;
    if (m_new > st.m_ref) st.m_ref = m_new;
    st.l *= alpha;
    sum2 = f2_fma(sum2, f2_pack(alpha, alpha), f2_pack(0.f, 0.f));
    if (st.o_valid) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(st.t_o + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(st.t_o + 32 * c, r);
        }
    }
#pragma unroll 1
    for (int c = 0; c < n_pcols; c += 16) {
        uint32_t r[16];
        tmem_ld16(t_p0 + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            if (F8) {
                float a0, a1, a2, a3;
                unpack_e4m3x2(static_cast<uint16_t>(r[e] & 0xFFFFu), a0, a1);
                unpack_e4m3x2(static_cast<uint16_t>(r[e] >> 16), a2, a3);
                r[e] = pack_e4m3x4(a0 * alpha, a1 * alpha, a2 * alpha, a3 * alpha);
            } else {
                const float lo = __uint_as_float(r[e] << 16) * alpha;
                const float hi = __uint_as_float(r[e] & 0xFFFF0000u) * alpha;
                r[e] = pack_bf16x2(lo, hi);
            }
        }
        tmem_st16(t_p0 + c, r);
    }
    tmem_st_wait();
}

// One pass over this thread's row of S: P = 2^(s * scale + bias - m_ref)
// (zero where masked out) in place over S in tensor memory (the P of chunk c
// goes to columns [16c, 16c+16) for bf16, [8c, 8c+8) for e4m3, while the only
// loads in flight cover [32(c+1), 32(c+3))).  Before a pair of 32-column chunks is
// written its maximum is checked against the reference; if it exceeds it by
// more than the headroom the reference moves first.  Returns the fp32 row
// sum of the tile.
template <int BLK, int HD, bool MASKED, bool F8>
__device__ __forceinline__ float tile_softmax(uint32_t t_s, int kind, int tok,
                                              const TileWalk<BLK>& walk, int j, float scale,
                                              float bias, float lpf, float inv_pfac, RowState& st) {
    constexpr int NC = BLK / 32;
    constexpr int kPColsPerChunk = F8 ? 8 : 16;   // TMEM columns of P per 32 keys
    constexpr float kHeadroom = Cfg<HD, BLK, F8>::kHeadroom;
    const uint64_t scale2 = f2_pack(scale, scale);
    const float pbias = F8 ? bias + lpf : bias;   // shift of the P written
    uint64_t shift2 = f2_pack(pbias - st.m_ref, pbias - st.m_ref);
    uint64_t sum2 = f2_pack(0.f, 0.f);
    uint32_t ra[32], rb[32];
    tmem_ld32(t_s, ra);
    tmem_ld32(t_s + 32, rb);
#pragma unroll 1
    for (int c = 0; c < NC; c += 2) {
        tmem_ld_wait();
        const uint32_t vba = chunk_bits<BLK, MASKED>(kind, tok, walk, j, c);
        const uint32_t vbb = chunk_bits<BLK, MASKED>(kind, tok, walk, j, c + 1);
        const float cm = fmaf(fmaxf(max32<MASKED>(ra, vba), max32<MASKED>(rb, vbb)), scale, bias);
        const bool need = cm > st.m_ref + kHeadroom;
        if (__any_sync(0xffffffffu, need)) {
            move_reference<HD, F8>(st, need ? cm : st.m_ref, sum2, t_s, kPColsPerChunk * c);
            shift2 = f2_pack(pbias - st.m_ref, pbias - st.m_ref);
        }
        p32<MASKED, F8>(ra, vba, t_s + kPColsPerChunk * c, scale2, shift2, sum2);
        if (c + 2 < NC) tmem_ld32(t_s + 32 * (c + 2), ra);
        p32<MASKED, F8>(rb, vbb, t_s + kPColsPerChunk * (c + 1), scale2, shift2, sum2);
        if (c + 3 < NC) tmem_ld32(t_s + 32 * (c + 3), rb);
    }
    tmem_st_wait();
    float a, b;
    f2_unpack(sum2, a, b);
    return F8 ? (a + b) * inv_pfac : a + b;
}

// ---------------------------------------------------------------------------
// softmax + correction + epilogue (warps 0-7)
// ---------------------------------------------------------------------------

template <int HD, int BLK, bool F8, bool CHUNK>
__device__ void softmax_wg(const AttnParams& P, Bars& B, uint8_t* smem, int m) {
    using C = Cfg<HD, BLK, F8>;
    const Dims& D = P.D;
    const int q4 = (threadIdx.x >> 5) & 3;        // TMEM lane quarter of this warp
    const int lane = threadIdx.x & 31;
    const int prow = 32 * q4 + lane;              // row of the 128-row query tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * q4) << 16;
    const uint32_t t_s = B.tmem_base + lane_off + (m == 0 ? C::kColS0 : C::kColS1);
    const uint32_t t_o = B.tmem_base + lane_off + (m == 0 ? C::kColO0 : C::kColO1);
    const float scale = 1.4426950408889634f / sqrtf((float)HD);   // log2(e) / sqrt(d)
    const float pseudo_bias = log2f((float)BLK);                   // ln n_j in log2 units
    uint32_t scnt = 0, ocnt = 0;

    for (int64_t w = blockIdx.x; w < P.n_slots; w += gridDim.x) {
        const int64_t o = sched_index(w, P.zigzag);
        if (o >= P.n_items) continue;
        const Item it = decode_item(P, o);
        if (!it.ok) continue;
        if (m == 1 && !it.has_m1) continue;
        TileWalk<BLK> walk;
        walk.init(P, it);
        if (walk.count() == 0) continue;   // a split without tiles
        const int split_slot = it.S > 1 ? it.slot + it.k : -1;   // scratch slot of a split
        const int mt = 2 * it.mp + m;
        const int pr = kTileM * mt + prow;
        const int hl = pr / BLK;
        const int tok = pr % BLK;
        const int h = it.g * D.G + hl;
        const int pos = it.i * BLK + tok;
        const int qoff = CHUNK ? P.q_off[it.s] : 0;
        bool row_valid = pos < it.L && (!CHUNK || pos >= qoff);
        const int64_t qtok = CHUNK ? (int64_t)P.cu_q[it.s] - qoff : it.tok0;   // q token of position 0
        RowState st{-INFINITY, 0.f, t_o, false};
        // e4m3: the logit scale folds in the Q scale of this row's block and
        // head; P' = P s_V K_row with K_row = 448 / (2^8 max s_V) over the
        // sequence and kv-head (so P' <= 448), undone in the epilogue.
        float q_sc = 1.f, k_row = 1.f;
        if (F8) {
            q_sc = __ldg(P.q_scale + (int64_t)(it.b0 + it.i) * D.Hq + h);
            k_row = 448.0f / (256.0f * __ldg(P.vmax + (int64_t)it.s * D.Hkv + it.g));
        }

        int kind, j, n = 0;
        while (walk.next(kind, j)) {
            float tscale = scale, pfac = 1.f, lpf = 0.f, inv_pfac = 1.f;
            if (F8) {
                // per-tile K and V scales: the block's, or a pseudo tile's chunk;
                // loaded before the S wait, which hides their latency
                const int64_t sb = (int64_t)it.b0 + (kind == kPseudo ? (int64_t)BLK * j : j);
                const float* ks = kind == kPseudo ? P.kbar_scale : P.k_scale;
                const float* vs = kind == kPseudo ? P.vbar_scale : P.v_scale;
                tscale = scale * q_sc * __ldg(ks + sb * D.Hkv + it.g);
                pfac = __ldg(vs + sb * D.Hkv + it.g) * k_row;
            }
            if (!warp_wait(&B.s_full[m], scnt & 1, B, P.status)) return;
            ++scnt;
            tc_fence_after();
            const bool masked = kind != kFull;
            const float bias = kind == kPseudo ? pseudo_bias : 0.f;
            if (F8) {
                lpf = __log2f(pfac);
                inv_pfac = __frcp_rn(pfac);
            }
            const float rsum =
                masked ? tile_softmax<BLK, HD, true, F8>(t_s, kind, tok, walk, j, tscale, bias, lpf,
                                                         inv_pfac, st)
                       : tile_softmax<BLK, HD, false, F8>(t_s, kind, tok, walk, j, tscale, bias, lpf,
                                                          inv_pfac, st);
            st.o_valid = true;
            st.l += rsum;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B.p_full[m]);
            ++n;
        }

        // epilogue: O / l as bf16, LSE = ln(l) + m_ref * ln 2; a split row
        // writes its part's O / l in fp32 and log2(l) + m_ref to its slot
        if (!warp_wait(&B.o_full[m], ocnt & 1, B, P.status)) return;
        ++ocnt;
        tc_fence_after();
        const float inv_l = 1.0f / (st.l * k_row);
        const bool split = split_slot >= 0;
        const int64_t srow = (int64_t)split_slot * (D.G * BLK) + pr;
        const int64_t orow = (qtok + pos) * D.Hq_str + h;
        if (row_valid && !(split ? FP2_CHECK(srow < P.n_split_rows, P.status)
                                 : FP2_CHECK(qtok + pos >= 0 && qtok + pos < P.Tq, P.status)))
            row_valid = false;
        char* dst = split ? reinterpret_cast<char*>(P.split_o + srow * HD)
                          : reinterpret_cast<char*>(P.o + orow * HD);
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(t_o + 32 * c, r);
            tmem_ld_wait();
            if (row_valid && split) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    reinterpret_cast<float4*>(dst)[(32 * c + e) / 4] =
                        make_float4(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                    __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
            } else if (row_valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                    reinterpret_cast<uint4*>(dst)[(32 * c + e) / 8] = v;
                }
            }
        }
        const float lse2 = st.m_ref + log2f(st.l);
        if (row_valid && split) P.split_lse[srow] = lse2;
        else if (row_valid) P.lse[(int64_t)h * (CHUNK ? P.Tq : D.T) + qtok + pos] = lse2 * 0.6931471805599453f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.o_free[m]);
    }
}

template <int HD, int BLK, bool F8, bool CHUNK>
__global__ void __launch_bounds__(kThreads, 1)
k_attn(const __grid_constant__ AttnParams P, const __grid_constant__ CUtensorMap tm_q,
       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
       const __grid_constant__ CUtensorMap tm_kbar, const __grid_constant__ CUtensorMap tm_vbar,
       const __grid_constant__ CUtensorMap tm_kbar_lo) {
    using C = Cfg<HD, BLK, F8>;
    if (!*P.meta_valid) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Bars& B = *reinterpret_cast<Bars*>(smem + C::kOffBar);
    const int warp = warp_id();
    const int lane = lane_id();

    if (threadIdx.x == 0) {
        for (int m = 0; m < 2; ++m) {
            mbar_init(&B.q_full[m], 1);
            mbar_init(&B.q_empty[m], 1);
            mbar_init(&B.s_full[m], 1);
            mbar_init(&B.p_full[m], kTileM / 32);
            mbar_init(&B.o_full[m], 1);
            mbar_init(&B.o_free[m], kTileM / 32);
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(&B.kv_full[s], 1);
            mbar_init(&B.kv_empty[s], 1);
        }
        mbar_init(&B.drain, 1);
        B.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) tmem_alloc(&B.tmem_base, C::kTmemCols);
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_kbar);
        if (F8) tma_prefetch_desc(&tm_kbar_lo);
        tma_prefetch_desc(&tm_vbar);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < 8) {
        softmax_wg<HD, BLK, F8, CHUNK>(P, B, smem, warp >> 2);
    } else if (warp == kProducerWarp) {
        if (lane == 0) producer<HD, BLK, F8, CHUNK>(P, B, smem, &tm_q, &tm_k, &tm_v, &tm_kbar, &tm_vbar,
                                                    &tm_kbar_lo);
    } else {
        if (lane == 0) mma_issuer<HD, BLK, F8>(P, B, smem);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(B.tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// merge of split rows
// ---------------------------------------------------------------------------

constexpr int kCombineThreads = 256;
constexpr int kCombineRows = 32;   // query rows per CTA (4 per warp)

// Grid (row split slot, query-tile pair x row chunk).  The CTAs of a split
// row's first slot merge kCombineRows of its query rows each: a row's
// non-empty splits k give lse = log2 sum_k 2^lse_k and
// O = sum_k 2^(lse_k - lse) O_k (one split per lane for the weights, the
// head dimension across the lanes for O); O goes out as bf16, LSE in
// natural-log units.  The other slots' CTAs return at once.
template <int HD, int BLK>
__global__ void __launch_bounds__(kCombineThreads) k_combine(const __grid_constant__ AttnParams P) {
    if (!*P.meta_valid) return;
    const int slot = blockIdx.x;
    const int64_t first = __ldg(P.slot_item + slot);
    if (__ldg(P.sched + first).w != slot) return;
    constexpr int kChunks = 2 * kTileM / kCombineRows;
    const int mp = blockIdx.y / kChunks;
    if (!FP2_CHECK(first >= 0 && first + mp < P.n_items, P.status)) return;
    const Item it = decode_item(P, first + mp);
    if (!it.ok) return;
    const Dims& D = P.D;
    int n;   // tiles of the whole row, as the attention roles walked them
    {
        Item whole = it;
        whole.S = 1;
        TileWalk<BLK> walk;
        walk.init(P, whole);
        n = walk.count();
    }
    constexpr int E = HD / 32;   // elements per lane
    const int lane = threadIdx.x & 31;
    const int64_t gb = (int64_t)D.G * BLK;
    const int r0 = (blockIdx.y % kChunks) * kCombineRows + (threadIdx.x >> 5) * (kCombineRows / 8);
    for (int rr = r0; rr < r0 + kCombineRows / 8; ++rr) {
        if (2 * it.mp + rr / kTileM >= P.n_mtiles) break;
        const int pr = 2 * it.mp * kTileM + rr;
        const int tok = pr % BLK;
        const int h = it.g * D.G + pr / BLK;
        const int pos = it.i * BLK + tok;
        const int qoff = P.q_off[it.s];
        if (pos >= it.L || pos < qoff) continue;
        const int64_t qtok = (int64_t)P.cu_q[it.s] - qoff;
        // lane k holds split k's log-sum-exp (-inf when the split had no tile)
        const bool live = lane < it.S && split_nonempty(lane, it.S, n) &&
                          FP2_CHECK((it.slot + lane + 1) * gb <= P.n_split_rows, P.status);
        const float lk = live ? P.split_lse[(it.slot + lane) * gb + pr] : -INFINITY;
        float mx = lk;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float wk = live ? exp2f(lk - mx) : 0.f;
        float wsum = wk;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        float acc[E];
#pragma unroll
        for (int x = 0; x < E; ++x) acc[x] = 0.f;
        for (int k = 0; k < it.S; ++k) {
            const float w = __shfl_sync(0xffffffffu, wk, k);
            if (w == 0.f) continue;
            const float* src = P.split_o + ((it.slot + k) * gb + pr) * HD + lane * E;
            if constexpr (E == 4) {
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
        const float inv = 1.0f / wsum;
        uint16_t* orow = P.o + ((qtok + pos) * D.Hq_str + h) * HD + lane * E;
        if constexpr (E == 4) {
            uint2 v;
            v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
            v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
            *reinterpret_cast<uint2*>(orow) = v;
        } else {
            *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        }
        if (lane == 0) P.lse[(int64_t)h * P.Tq + qtok + pos] = (mx + log2f(wsum)) * 0.6931471805599453f;
    }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

// Largest V scale of every (sequence, kv-head): over the blocks' V scales and
// the chunk scales of the e4m3 V block means (FP8 path).
__global__ void __launch_bounds__(256) k_vmax(Dims D, PlanPtrs P, const float* __restrict__ v_scale) {
    if (!*P.meta_valid) return;
    const int s = blockIdx.x, g = blockIdx.y;
    const int b0 = P.cu_blocks[s], b1 = P.cu_blocks[s + 1];
    float mx = 0.f;
    for (int b = b0 + threadIdx.x; b < b1; b += blockDim.x) {
        mx = fmaxf(mx, v_scale[(int64_t)b * D.Hkv + g]);
        if ((b - b0) % D.B == 0) mx = fmaxf(mx, P.vbar_scale[(int64_t)b * D.Hkv + g]);
    }
    __shared__ float red[8];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
        P.vmax[(int64_t)s * D.Hkv + g] = mx > 0.f ? mx : 1.0f;
    }
}

template <int HD, int BLK, bool F8>
int launch_attn_t(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* q,
                  const void* k, const void* v, const float* qs, const float* ks, const float* vs,
                  void* o, float* lse, uint32_t flags, cudaStream_t st) {
    using C = Cfg<HD, BLK, F8>;
    const Dims& D = L.dims;
    const cuuint64_t eb = C::kElt;                         // bytes per element
    const cuuint32_t ae = C::kAtomElems;                   // elements per 128-byte atom row
    CUtensorMap tq, tk, tv, tkb, tvb, tkb_lo;
    {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hq, (cuuint64_t)L.Tq};
        cuuint64_t str[2] = {(cuuint64_t)HD * eb, (cuuint64_t)D.Hq_str * HD * eb};
        cuuint32_t box[3] = {ae, 1, (cuuint32_t)BLK};
        if (!make_tensor_map(&tq, q, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
    }
    if (D.page_size == 0) {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, (cuuint64_t)D.T};
        cuuint64_t str[2] = {(cuuint64_t)HD * eb, (cuuint64_t)D.Hkv_str * HD * eb};
        cuuint32_t box[3] = {ae, 1, (cuuint32_t)BLK};
        if (!make_tensor_map(&tk, k, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
        if (!make_tensor_map(&tv, v, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
    } else {
        cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, 64, (cuuint64_t)D.num_pages};
        cuuint64_t str[3] = {(cuuint64_t)HD * eb, (cuuint64_t)D.Hkv_str * HD * eb,
                             (cuuint64_t)64 * D.Hkv_str * HD * eb};
        cuuint32_t box[4] = {ae, 1, 64, 1};
        if (!make_tensor_map(&tk, k, 4, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
        if (!make_tensor_map(&tv, v, 4, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, (cuuint64_t)D.NB};
        cuuint64_t str[2] = {(cuuint64_t)HD * eb, (cuuint64_t)D.Hkv * HD * eb};
        cuuint32_t box[3] = {ae, 1, (cuuint32_t)BLK};
        const void* kb = F8 ? static_cast<const void*>(pp.kbar8) : static_cast<const void*>(pp.kbar16);
        const void* vb = F8 ? static_cast<const void*>(pp.vbar8) : static_cast<const void*>(pp.vbar16);
        if (!make_tensor_map(&tkb, kb, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
        if (!make_tensor_map(&tvb, vb, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
        // the second e4m3 term of the key means (e4m3 only; unused for bf16)
        const void* kl = F8 ? static_cast<const void*>(pp.kbar8lo) : kb;
        if (!make_tensor_map(&tkb_lo, kl, 3, dims, str, box, F8 ? kMapU8 : kMapBF16)) return FP2_ERR_CUDA;
    }
    AttnParams P;
    P.D = D;
    P.cu_seqlens = p->cu_seqlens;
    P.page_table = p->page_table;
    P.row_ptr = pp.row_ptr;
    P.col_idx = pp.col_idx;
    P.kept_mask = pp.kept_mask;
    P.block_seq = pp.block_seq;
    P.cu_blocks = pp.cu_blocks;
    P.meta_valid = pp.meta_valid;
    P.status = pp.status;
    P.o = static_cast<uint16_t*>(o);
    P.lse = lse;
    P.q_scale = qs;
    P.k_scale = ks;
    P.v_scale = vs;
    P.kbar_scale = pp.kbar_scale;
    P.vbar_scale = pp.vbar_scale;
    P.vmax = pp.vmax;
    P.flags = flags;
    const SchedDims& S = L.sched;
    P.n_mtiles = S.n_mtiles;
    P.n_items = S.n_items;
    P.sched = pp.sched;
    P.split_o = pp.split_o;
    P.split_lse = pp.split_lse;
    P.slot_item = pp.slot_item;
    P.cu_q = L.chunked ? p->cu_q_seqlens : p->cu_seqlens;
    P.q_off = pp.q_off;
    P.Tq = L.Tq;
    const int sms = sm_count();
    if (sms <= 0) return FP2_ERR_CUDA;
    const int64_t grid = S.n_items < sms ? S.n_items : sms;
    P.n_slots = (S.n_items + grid - 1) / grid * grid;
    P.n_split_rows = S.split_slots * D.Hkv * D.G * BLK;
    P.zigzag = P.n_slots / grid <= kZigZagMaxPasses;
    auto kernel = L.chunked ? k_attn<HD, BLK, F8, true> : k_attn<HD, BLK, F8, false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
        return FP2_ERR_CUDA;
    if (F8) k_vmax<<<dim3(D.n_seqs, D.Hkv), 256, 0, st>>>(D, pp, vs);
    kernel<<<(unsigned)grid, kThreads, C::kSmemBytes, st>>>(P, tq, tk, tv, tkb, tvb, tkb_lo);
    if (S.split_slots > 0)
        k_combine<HD, BLK><<<dim3((unsigned)(S.split_slots * D.Hkv), S.n_pairs * (2 * kTileM / kCombineRows)),
                             kCombineThreads, 0, st>>>(P);
    return cudaGetLastError() == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

}  // namespace

int launch_prefill(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* q,
                   const void* k, const void* v, const float* qs, const float* ks, const float* vs,
                   int dtype, void* o, float* lse, uint32_t flags, cudaStream_t st) {
    const Dims& D = L.dims;
    if (dtype == FP2_DTYPE_E4M3) {
        if (D.d != 128) return FP2_ERR_UNSUPPORTED;   // e4m3 rows must fill 128-byte atoms
        if (D.B == 128) return launch_attn_t<128, 128, true>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
        return launch_attn_t<128, 64, true>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
    }
    if (D.d == 128 && D.B == 128)
        return launch_attn_t<128, 128, false>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
    if (D.d == 128 && D.B == 64)
        return launch_attn_t<128, 64, false>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
    if (D.d == 64 && D.B == 128)
        return launch_attn_t<64, 128, false>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
    return launch_attn_t<64, 64, false>(L, p, pp, q, k, v, qs, ks, vs, o, lse, flags, st);
}

}  // namespace fp2
