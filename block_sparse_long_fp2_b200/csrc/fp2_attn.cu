// Stage 2 of FlashPrefill V2 (Figure 3 / Figure 4 of the metallab.ai summary
// of arXiv 2608.19758): sparse attention over the selected key blocks with
// the mean correction merged into the same online softmax.
//
// One persistent CTA per SM (320 threads) walks work items longest row
// first.  A work item is one CSR row (sequence s, kv-head g, query block i)
// restricted to two PackGQA query tiles of 128 rows each (the G heads x B
// tokens of the row, packed head-major).  Both tiles share every K/V tile
// the CTA streams, so K/V cross HBM once per kv-head (PackGQA).
//
// Roles (warp specialisation):
//   warps 0-3   softmax warpgroup of query tile 0 (TMEM lanes 0-127)
//   warps 4-7   softmax warpgroup of query tile 1
//   warp 8      TMA producer: Q tiles, then per kept block its K and V tiles
//               (through the page table when paged), then per pseudo tile
//               up to B bf16 block means Kbar/Vbar; a ring of 3 K-or-V slots.
//   warp 9      allocates tensor memory and issues tcgen05 MMAs:
//               S_m = Q_m K^T into TMEM, O_m += P_m V into TMEM.
// Issue order for K/V tile n:  S0(n), PV1(n-1), S1(n), PV0(n).  Every commit
// that publishes S_m(n) therefore also covers PV_m(n-1), so the softmax
// warps may rescale O_m and overwrite their P buffer as soon as S_m(n) is
// visible.
//
// Mean correction (Figure 4): each skipped, fully visible block j adds one
// pseudo-key with key Kbar_j, value Vbar_j and logit bias ln n_j = ln B.
// Up to B skipped blocks form one pseudo tile, run through exactly the same
// MMA + softmax path as a real K/V tile, with the columns of kept blocks
// (and of blocks j >= i) masked out.
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
constexpr int kMmaWarp = 9;
constexpr int kSlots = 3;

constexpr int pow2_ceil(int x) {
    int p = 32;
    while (p < x) p <<= 1;
    return p;
}

template <int HD, int BLK>
struct Cfg {
    static constexpr int kQBytes = kTileM * HD * 2;      // one 128-row query tile (bf16)
    static constexpr int kSlotBytes = BLK * HD * 2;      // one K or V tile (bf16)
    static constexpr int kOffQ = 0;
    static constexpr int kOffSlot = 2 * kQBytes;
    static constexpr int kOffBar = kOffSlot + kSlots * kSlotBytes;
    static constexpr int kSmemBytes = kOffBar + 512 + 1024;   // barriers + alignment slack
    static constexpr int kColS0 = 0;
    static constexpr int kColS1 = BLK;
    static constexpr int kColO0 = 2 * BLK;
    static constexpr int kColO1 = 2 * BLK + HD;
    static constexpr int kTmemCols = pow2_ceil(2 * (BLK + HD));
    static constexpr int kAtomQ = kTileM * 128;          // bytes between 64-column atoms of Q
    static constexpr int kAtomKV = BLK * 128;            // bytes between 64-column atoms of K / V
};

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[kSlots], kv_empty[kSlots];
    uint64_t s_full[2], s_free[2];
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
    uint32_t flags;
    int n_mtiles;   // 128-row query tiles per row = G * B / 128
    int n_pairs;    // work items per row = ceil(n_mtiles / 2)
    int64_t n_items;
};

// One work item: row (s, g, i) and query tiles 2*mp, 2*mp+1.
struct Item {
    int s, g, i, mp;
    int64_t b, r;
    int kbeg, kend;      // CSR range of the row
    int tok0, L;         // first token of the sequence, its length
    int b0;              // first global block of the sequence
    bool has_m1;
};

__device__ __forceinline__ Item decode_item(const AttnParams& P, int64_t w) {
    Item it;
    const int64_t rank = w / P.n_pairs;
    it.mp = (int)(w % P.n_pairs);
    it.b = P.D.NB - 1 - rank / P.D.Hkv;       // latest query blocks first (longest rows)
    it.g = (int)(rank % P.D.Hkv);
    it.s = P.block_seq[it.b];
    it.b0 = P.cu_blocks[it.s];
    it.i = (int)(it.b - it.b0);
    it.r = (int64_t)it.g * P.D.NB + it.b;
    it.kbeg = P.row_ptr[it.r];
    it.kend = P.row_ptr[it.r + 1];
    it.tok0 = P.cu_seqlens[it.s];
    it.L = P.cu_seqlens[it.s + 1] - it.tok0;
    it.has_m1 = 2 * it.mp + 1 < P.n_mtiles;
    return it;
}

enum TileKind { kFull = 0, kDiag = 1, kPseudo = 2 };

// Walks the tiles of an item: the kept blocks in CSR order, then the pseudo
// tiles that contain at least one skipped block.  Every role runs the same
// walk, so they agree on the sequence without exchanging it.
template <int BLK>
struct TileWalk {
    static constexpr int W = BLK / 32;
    const int32_t* cols;
    const uint32_t* mask;
    int n_kept, t, i, pt, n_pt, mask_words;

    __device__ __forceinline__ void init(const AttnParams& P, const Item& it) {
        cols = P.col_idx + it.kbeg;
        n_kept = it.kend - it.kbeg;
        t = 0;
        i = it.i;
        mask = P.kept_mask + it.r * P.D.mask_words;
        mask_words = P.D.mask_words;
        pt = 0;
        n_pt = (P.flags & FP2_NO_CORRECTION) ? 0 : (it.i + BLK - 1) / BLK;
    }
    // skip bits of blocks BLK*pt + 32*w .. +31 (skipped = visible, j < i, not kept)
    __device__ __forceinline__ uint32_t skip_word(int p, int w) const {
        const int j0 = BLK * p + 32 * w;
        if (j0 >= i) return 0u;
        const uint32_t valid = (j0 + 32 <= i) ? 0xFFFFFFFFu : ((1u << (i - j0)) - 1u);
        const int widx = j0 / 32;
        const uint32_t kept = widx < mask_words ? mask[widx] : 0xFFFFFFFFu;
        return ~kept & valid;
    }
    __device__ __forceinline__ bool has_skip(int p) const {
        uint32_t any = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) any |= skip_word(p, w);
        return any != 0;
    }
    // Advances to the next tile; returns false at the end.
    __device__ __forceinline__ bool next(int& kind, int& j) {
        if (t < n_kept) {
            j = cols[t++];
            kind = (j == i) ? kDiag : kFull;
            return true;
        }
        while (pt < n_pt && !has_skip(pt)) ++pt;
        if (pt >= n_pt) return false;
        j = pt++;
        kind = kPseudo;
        return true;
    }
    __device__ __forceinline__ bool is_last() {
        if (t < n_kept) return false;
        int p = pt;
        while (p < n_pt && !has_skip(p)) ++p;
        return p >= n_pt;
    }
};

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

template <int HD, int BLK>
__device__ void producer(const AttnParams& P, Bars& B, uint8_t* smem, const CUtensorMap* tm_q,
                         const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_kbar, const CUtensorMap* tm_vbar) {
    using C = Cfg<HD, BLK>;
    const Dims& D = P.D;
    uint32_t qcnt[2] = {0, 0}, qloaded[2] = {0, 0};
    uint32_t ld = 0;                 // K/V loads issued (slot = ld % 3)
    uint32_t issued[kSlots] = {0, 0, 0};
    const bool paged = D.page_size != 0;
    for (int64_t w = blockIdx.x; w < P.n_items; w += gridDim.x) {
        const Item it = decode_item(P, w);
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
                for (int a = 0; a < HD / 64; ++a)
                    tma_load_3d(qdst + a * C::kAtomQ + ht * BLK * 128, tm_q, &B.q_full[m], 64 * a,
                                it.g * D.G + hl, it.tok0 + it.i * BLK);
            }
        }
        TileWalk<BLK> walk;
        walk.init(P, it);
        int kind, j;
        while (walk.next(kind, j)) {
            for (int kv = 0; kv < 2; ++kv) {
                const int slot = ld % kSlots;
                const uint32_t use = ld / kSlots;
                if (!mbar_wait(&B.kv_empty[slot], (use & 1) ^ 1, &B.abort, P.status)) goto drain;
                ++ld;
                issued[slot] = use + 1;
                uint64_t* bar = &B.kv_full[slot];
                mbar_arrive_expect_tx(bar, C::kSlotBytes);
                uint8_t* dst = smem + C::kOffSlot + slot * C::kSlotBytes;
                if (kind == kPseudo) {
                    const CUtensorMap* tm = kv == 0 ? tm_kbar : tm_vbar;
#pragma unroll
                    for (int a = 0; a < HD / 64; ++a)
                        tma_load_3d(dst + a * C::kAtomKV, tm, bar, 64 * a, it.g, it.b0 + j * BLK);
                } else if (!paged) {
                    const CUtensorMap* tm = kv == 0 ? tm_k : tm_v;
#pragma unroll
                    for (int a = 0; a < HD / 64; ++a)
                        tma_load_3d(dst + a * C::kAtomKV, tm, bar, 64 * a, it.g, it.tok0 + j * BLK);
                } else {
                    const CUtensorMap* tm = kv == 0 ? tm_k : tm_v;
                    const int n_pages_s = (it.L + 63) / 64;
#pragma unroll
                    for (int pg = 0; pg < BLK / 64; ++pg) {
                        const int pi = (j * BLK) / 64 + pg;
                        int id = D.num_pages;   // out of range: the copy fills zeros
                        if (pi < n_pages_s) {
                            const int e = P.page_table[(int64_t)it.s * D.pt_stride + pi];
                            if (e >= 0 && e < D.num_pages) id = e;
                            else atomicOr(P.status, (int32_t)FP2_STATUS_BAD_PAGE);
                        }
#pragma unroll
                        for (int a = 0; a < HD / 64; ++a)
                            tma_load_4d(dst + a * C::kAtomKV + pg * 64 * 128, tm, bar, 64 * a, it.g,
                                        0, id);
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

template <int HD, int BLK>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr) {
    using C = Cfg<HD, BLK>;
    constexpr uint32_t idesc = idesc_bf16(kTileM, BLK, false);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t a = q_addr + (kk / 4) * C::kAtomQ + (kk % 4) * 32;
        const uint32_t b = k_addr + (kk / 4) * C::kAtomKV + (kk % 4) * 32;
        umma_f16(tmem_s, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(b, 16, 1024), idesc,
                 kk > 0 ? 1u : 0u);
    }
}

template <int HD, int BLK>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr,
                                         bool accumulate) {
    using C = Cfg<HD, BLK>;
    constexpr uint32_t idesc = idesc_bf16(kTileM, HD, true);
#pragma unroll
    for (int kk = 0; kk < BLK / 16; ++kk) {
        const uint32_t b = v_addr + kk * 16 * 128;
        umma_f16_ts(tmem_o, tmem_p + kk * 8, smem_desc_sw128(b, C::kAtomKV, 1024), idesc,
                    (accumulate || kk > 0) ? 1u : 0u);
    }
}

struct PrevTile {
    bool valid, has_m1, first, last;
    int vslot;
};

template <int HD, int BLK>
__device__ void mma_issuer(const AttnParams& P, Bars& B, uint8_t* smem) {
    using C = Cfg<HD, BLK>;
    const uint32_t tb = B.tmem_base;
    const uint32_t s_base = smem_u32(smem);
    const uint32_t q_addr[2] = {s_base + C::kOffQ, s_base + C::kOffQ + C::kQBytes};
    const uint32_t t_s[2] = {tb + C::kColS0, tb + C::kColS1};
    const uint32_t t_o[2] = {tb + C::kColO0, tb + C::kColO1};
    uint32_t qcnt[2] = {0, 0}, scnt[2] = {0, 0}, pcnt[2] = {0, 0}, ocnt[2] = {0, 0};
    uint32_t ld = 0;
    PrevTile prev{false, false, false, false, 0};

    auto pv1 = [&](const PrevTile& pt) -> bool {
        if (!mbar_wait(&B.p_full[1], pcnt[1] & 1, &B.abort, P.status)) return false;
        ++pcnt[1];
        if (pt.first && !mbar_wait(&B.o_free[1], (ocnt[1] & 1) ^ 1, &B.abort, P.status)) return false;
        tc_fence_after();
        issue_pv<HD, BLK>(t_o[1], t_s[1], s_base + C::kOffSlot + pt.vslot * C::kSlotBytes,
                          !pt.first);
        umma_commit(&B.kv_empty[pt.vslot]);
        if (pt.last) {
            umma_commit(&B.o_full[1]);
            ++ocnt[1];
        }
        return true;
    };

    for (int64_t w = blockIdx.x; w < P.n_items; w += gridDim.x) {
        const Item it = decode_item(P, w);
        TileWalk<BLK> walk;
        walk.init(P, it);
        int kind, j, n = 0;
        while (walk.next(kind, j)) {
            const bool first = n == 0;
            const bool last = walk.is_last();
            const int ks = ld % kSlots;
            const uint32_t kuse = ld / kSlots;
            ++ld;
            const int vs = ld % kSlots;
            const uint32_t vuse = ld / kSlots;
            ++ld;
            const uint32_t k_addr = s_base + C::kOffSlot + ks * C::kSlotBytes;
            const uint32_t v_addr = s_base + C::kOffSlot + vs * C::kSlotBytes;
            // S0 = Q0 K^T
            if (first) {
                if (!mbar_wait(&B.q_full[0], qcnt[0] & 1, &B.abort, P.status)) goto drain;
                ++qcnt[0];
            }
            if (!mbar_wait(&B.kv_full[ks], kuse & 1, &B.abort, P.status)) goto drain;
            if (!mbar_wait(&B.s_free[0], (scnt[0] & 1) ^ 1, &B.abort, P.status)) goto drain;
            tc_fence_after();
            issue_s<HD, BLK>(t_s[0], q_addr[0], k_addr);
            umma_commit(&B.s_full[0]);
            ++scnt[0];
            if (!it.has_m1) {
                umma_commit(&B.kv_empty[ks]);
                if (last) umma_commit(&B.q_empty[0]);
            }
            // PV1 of the previous tile
            if (prev.valid && prev.has_m1) {
                if (!pv1(prev)) goto drain;
            }
            // S1 = Q1 K^T
            if (it.has_m1) {
                if (first) {
                    if (!mbar_wait(&B.q_full[1], qcnt[1] & 1, &B.abort, P.status)) goto drain;
                    ++qcnt[1];
                }
                if (!mbar_wait(&B.s_free[1], (scnt[1] & 1) ^ 1, &B.abort, P.status)) goto drain;
                tc_fence_after();
                issue_s<HD, BLK>(t_s[1], q_addr[1], k_addr);
                umma_commit(&B.s_full[1]);
                ++scnt[1];
                umma_commit(&B.kv_empty[ks]);
                if (last) {
                    umma_commit(&B.q_empty[0]);
                    umma_commit(&B.q_empty[1]);
                }
            }
            // PV0 of this tile
            if (!mbar_wait(&B.kv_full[vs], vuse & 1, &B.abort, P.status)) goto drain;
            if (!mbar_wait(&B.p_full[0], pcnt[0] & 1, &B.abort, P.status)) goto drain;
            ++pcnt[0];
            if (first && !mbar_wait(&B.o_free[0], (ocnt[0] & 1) ^ 1, &B.abort, P.status)) goto drain;
            tc_fence_after();
            issue_pv<HD, BLK>(t_o[0], t_s[0], v_addr, !first);
            if (!it.has_m1) umma_commit(&B.kv_empty[vs]);
            if (last) {
                umma_commit(&B.o_full[0]);
                ++ocnt[0];
            }
            prev = PrevTile{true, it.has_m1, first, last, vs};
            ++n;
        }
    }
    if (prev.valid && prev.has_m1) pv1(prev);
drain:
    // Wait until every MMA issued above has completed.
    umma_commit(&B.drain);
    mbar_wait_drain(&B.drain, 0, P.status);
}

// Row maximum of the raw (unscaled) scores of the masked-in columns of this
// thread's row of S.  Two 32-column TMEM loads in flight.
template <int BLK, bool MASKED>
__device__ __forceinline__ uint32_t chunk_bits(int kind, int tok, const TileWalk<BLK>& walk, int j,
                                               int c32) {
    return MASKED ? col_bits(kind, tok, walk, j, c32) : 0xFFFFFFFFu;
}

template <bool MASKED>
__device__ __forceinline__ void max32(const uint32_t (&r)[32], uint32_t vb, float& mx) {
    if (MASKED) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if ((vb >> e) & 1u) mx = fmaxf(mx, __uint_as_float(r[e]));
    } else {
#pragma unroll
        for (int e = 0; e < 32; e += 2) mx = fmax3(mx, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
    }
}

// Row maximum of the raw (unscaled) scores of the masked-in columns of this
// thread's row of S.  32-column TMEM loads, two in flight.
template <int BLK, bool MASKED>
__device__ __forceinline__ float tile_max(uint32_t t_s, int kind, int tok, const TileWalk<BLK>& walk,
                                          int j) {
    constexpr int NC = BLK / 32;
    float mx = -INFINITY;
    uint32_t ra[32], rb[32];
    tmem_ld32(t_s, ra);
    tmem_ld32(t_s + 32, rb);
#pragma unroll 1
    for (int c = 0; c < NC; c += 2) {
        tmem_ld_wait();
        max32<MASKED>(ra, chunk_bits<BLK, MASKED>(kind, tok, walk, j, c), mx);
        if (c + 2 < NC) tmem_ld32(t_s + 32 * (c + 2), ra);
        max32<MASKED>(rb, chunk_bits<BLK, MASKED>(kind, tok, walk, j, c + 1), mx);
        if (c + 3 < NC) tmem_ld32(t_s + 32 * (c + 3), rb);
    }
    return mx;
}

// 32 columns of P = 2^(s * scale + shift) as 16 packed bf16 pairs, written
// into tensor memory over the first half of the 32 S columns just read
// (P of keys 2c and 2c+1 in column c): the A operand of the P.V MMA.
template <bool MASKED>
__device__ __forceinline__ void p32(const uint32_t (&r)[32], uint32_t vb, uint32_t t_p,
                                    uint64_t scale2, uint64_t shift2, uint64_t& sum2) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t packed[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
            const int e = 16 * h + 2 * e2;
            float s0 = __uint_as_float(r[e]), s1 = __uint_as_float(r[e + 1]);
            if (MASKED) {
                s0 = ((vb >> e) & 1u) ? s0 : -INFINITY;
                s1 = ((vb >> (e + 1)) & 1u) ? s1 : -INFINITY;
            }
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s0, s1), scale2, shift2), x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            sum2 = f2_add(sum2, f2_pack(p0, p1));
            packed[e2] = pack_bf16x2(p0, p1);
        }
        tmem_st8(t_p + 8 * h, packed);
    }
}

// P = 2^(s * scale + shift) for this thread's row of S (zero where masked
// out), written as bf16 pairs in place over S in tensor memory (column c of
// the P operand holds keys 2c, 2c+1 and lies inside S columns already read:
// the P of chunk c goes to columns [16c, 16c+16) while the only loads in
// flight cover [32(c+1), 32(c+2))).  Returns the fp32 row sum.
template <int BLK, bool MASKED>
__device__ __forceinline__ float tile_p(uint32_t t_s, int kind, int tok, const TileWalk<BLK>& walk,
                                        int j, float scale, float shift) {
    constexpr int NC = BLK / 32;
    const uint64_t scale2 = f2_pack(scale, scale);
    const uint64_t shift2 = f2_pack(shift, shift);
    uint64_t sum2 = f2_pack(0.f, 0.f);
    uint32_t ra[32], rb[32];
    tmem_ld32(t_s, ra);
    tmem_ld32(t_s + 32, rb);
#pragma unroll 1
    for (int c = 0; c < NC; c += 2) {
        tmem_ld_wait();
        p32<MASKED>(ra, chunk_bits<BLK, MASKED>(kind, tok, walk, j, c), t_s + 16 * c, scale2, shift2,
                    sum2);
        if (c + 2 < NC) tmem_ld32(t_s + 32 * (c + 2), ra);
        p32<MASKED>(rb, chunk_bits<BLK, MASKED>(kind, tok, walk, j, c + 1), t_s + 16 * (c + 1), scale2,
                    shift2, sum2);
        if (c + 3 < NC) tmem_ld32(t_s + 32 * (c + 3), rb);
    }
    tmem_st_wait();
    float a, b;
    f2_unpack(sum2, a, b);
    return a + b;
}

// ---------------------------------------------------------------------------
// softmax + correction + epilogue (warps 0-7)
// ---------------------------------------------------------------------------

template <int HD, int BLK>
__device__ void softmax_wg(const AttnParams& P, Bars& B, uint8_t* smem, int m) {
    using C = Cfg<HD, BLK>;
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

    for (int64_t w = blockIdx.x; w < P.n_items; w += gridDim.x) {
        const Item it = decode_item(P, w);
        if (m == 1 && !it.has_m1) continue;
        const int mt = 2 * it.mp + m;
        const int pr = kTileM * mt + prow;
        const int hl = pr / BLK;
        const int tok = pr % BLK;
        const int h = it.g * D.G + hl;
        const int pos = it.i * BLK + tok;
        const bool row_valid = pos < it.L;
        float m_ref = -INFINITY, l = 0.f;

        TileWalk<BLK> walk;
        walk.init(P, it);
        int kind, j, n = 0;
        while (walk.next(kind, j)) {
            if (!warp_wait(&B.s_full[m], scnt & 1, B, P.status)) return;
            ++scnt;
            tc_fence_after();
            const bool masked = kind != kFull;
            const float bias = kind == kPseudo ? pseudo_bias : 0.f;
            // pass 1: row maximum of the masked scores
            const float rmax_raw = masked ? tile_max<BLK, true>(t_s, kind, tok, walk, j)
                                          : tile_max<BLK, false>(t_s, kind, tok, walk, j);
            const float rmax = fmaf(rmax_raw, scale, bias);   // -inf stays -inf
            if (n == 0) {
                m_ref = rmax;
            } else {
                // lazy rescale: O and l move to a new reference only when the
                // row maximum grew by more than 2^8
                const bool need = rmax > m_ref + 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = fmaxf(m_ref, rmax);
                    const float alpha = ex2_approx(m_ref - m_new);
                    m_ref = m_new;
                    l *= alpha;
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(t_o + 32 * c, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(t_o + 32 * c, r);
                    }
                    tmem_st_wait();
                }
            }
            // pass 2: P in place over S
            const float rsum = masked ? tile_p<BLK, true>(t_s, kind, tok, walk, j, scale, bias - m_ref)
                                      : tile_p<BLK, false>(t_s, kind, tok, walk, j, scale, bias - m_ref);
            l += rsum;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&B.s_free[m]);
                mbar_arrive(&B.p_full[m]);
            }
            ++n;
        }

        // epilogue: O / l as bf16, LSE = ln(l) + m_ref * ln 2
        if (!warp_wait(&B.o_full[m], ocnt & 1, B, P.status)) return;
        ++ocnt;
        tc_fence_after();
        const float inv_l = 1.0f / l;
        uint16_t* orow = P.o + ((int64_t)(it.tok0 + pos) * D.Hq + h) * HD;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(t_o + 32 * c, r);
            tmem_ld_wait();
            if (row_valid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[e + 0]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                    *reinterpret_cast<uint4*>(orow + 32 * c + e) = v;
                }
            }
        }
        if (row_valid) P.lse[(int64_t)h * D.T + it.tok0 + pos] = (m_ref + log2f(l)) * 0.6931471805599453f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.o_free[m]);
    }
}

template <int HD, int BLK>
__global__ void __launch_bounds__(kThreads, 1)
k_attn(const __grid_constant__ AttnParams P, const __grid_constant__ CUtensorMap tm_q,
       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
       const __grid_constant__ CUtensorMap tm_kbar, const __grid_constant__ CUtensorMap tm_vbar) {
    using C = Cfg<HD, BLK>;
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
            mbar_init(&B.s_free[m], kTileM / 32);
            mbar_init(&B.p_full[m], kTileM / 32);
            mbar_init(&B.o_full[m], 1);
            mbar_init(&B.o_free[m], kTileM / 32);
        }
        for (int s = 0; s < kSlots; ++s) {
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
        tma_prefetch_desc(&tm_vbar);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < 8) {
        softmax_wg<HD, BLK>(P, B, smem, warp >> 2);
    } else if (warp == kProducerWarp) {
        if (lane == 0) producer<HD, BLK>(P, B, smem, &tm_q, &tm_k, &tm_v, &tm_kbar, &tm_vbar);
    } else {
        if (lane == 0) mma_issuer<HD, BLK>(P, B, smem);
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
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 tensor map with 128-byte swizzle; dims innermost first, strides in
// bytes for dims 1..rank-1.
bool make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                     strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int HD, int BLK>
int launch_attn_t(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* q,
                  const void* k, const void* v, void* o, float* lse, uint32_t flags,
                  cudaStream_t st) {
    using C = Cfg<HD, BLK>;
    const Dims& D = L.dims;
    CUtensorMap tq, tk, tv, tkb, tvb;
    {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hq, (cuuint64_t)D.T};
        cuuint64_t str[2] = {(cuuint64_t)HD * 2, (cuuint64_t)D.Hq * HD * 2};
        cuuint32_t box[3] = {64, 1, (cuuint32_t)BLK};
        if (!make_map(&tq, q, 3, dims, str, box)) return FP2_ERR_CUDA;
    }
    if (D.page_size == 0) {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, (cuuint64_t)D.T};
        cuuint64_t str[2] = {(cuuint64_t)HD * 2, (cuuint64_t)D.Hkv * HD * 2};
        cuuint32_t box[3] = {64, 1, (cuuint32_t)BLK};
        if (!make_map(&tk, k, 3, dims, str, box)) return FP2_ERR_CUDA;
        if (!make_map(&tv, v, 3, dims, str, box)) return FP2_ERR_CUDA;
    } else {
        cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, 64, (cuuint64_t)D.num_pages};
        cuuint64_t str[3] = {(cuuint64_t)HD * 2, (cuuint64_t)D.Hkv * HD * 2,
                             (cuuint64_t)64 * D.Hkv * HD * 2};
        cuuint32_t box[4] = {64, 1, 64, 1};
        if (!make_map(&tk, k, 4, dims, str, box)) return FP2_ERR_CUDA;
        if (!make_map(&tv, v, 4, dims, str, box)) return FP2_ERR_CUDA;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)D.Hkv, (cuuint64_t)D.NB};
        cuuint64_t str[2] = {(cuuint64_t)HD * 2, (cuuint64_t)D.Hkv * HD * 2};
        cuuint32_t box[3] = {64, 1, (cuuint32_t)BLK};
        if (!make_map(&tkb, pp.kbar16, 3, dims, str, box)) return FP2_ERR_CUDA;
        if (!make_map(&tvb, pp.vbar16, 3, dims, str, box)) return FP2_ERR_CUDA;
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
    P.flags = flags;
    P.n_mtiles = D.G * BLK / kTileM;
    P.n_pairs = (P.n_mtiles + 1) / 2;
    P.n_items = D.R * P.n_pairs;
    const int sms = sm_count();
    if (sms <= 0) return FP2_ERR_CUDA;
    const int64_t grid = P.n_items < sms ? P.n_items : sms;
    if (cudaFuncSetAttribute(k_attn<HD, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
        return FP2_ERR_CUDA;
    k_attn<HD, BLK><<<(unsigned)grid, kThreads, C::kSmemBytes, st>>>(P, tq, tk, tv, tkb, tvb);
    return cudaGetLastError() == cudaSuccess ? FP2_OK : FP2_ERR_CUDA;
}

}  // namespace

int launch_prefill(const Layout& L, const fp2_problem* p, const PlanPtrs& pp, const void* q,
                   const void* k, const void* v, const float* qs, const float* ks, const float* vs,
                   int dtype, void* o, float* lse, uint32_t flags, cudaStream_t st) {
    (void)qs;
    (void)ks;
    (void)vs;
    if (dtype != FP2_DTYPE_BF16) return FP2_ERR_UNSUPPORTED;
    const Dims& D = L.dims;
    if (D.d == 128 && D.B == 128) return launch_attn_t<128, 128>(L, p, pp, q, k, v, o, lse, flags, st);
    if (D.d == 128 && D.B == 64) return launch_attn_t<128, 64>(L, p, pp, q, k, v, o, lse, flags, st);
    if (D.d == 64 && D.B == 128) return launch_attn_t<64, 128>(L, p, pp, q, k, v, o, lse, flags, st);
    return launch_attn_t<64, 64>(L, p, pp, q, k, v, o, lse, flags, st);
}

}  // namespace fp2
