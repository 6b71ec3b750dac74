// Indexer scoring on the tcgen05 tensor cores.
//
// One kernel scores 128 candidates per tile for one query row:
//     score(i, x) = sum_h w[i,h] * max(0, q[i,h,:] . x)
// (the lightning-indexer form HISA reuses for both stages: gptget.net
// summary, "Methodology" — block representatives and candidate tokens are
// scored by the same original indexer).  The dot products are one UMMA per
// 16-wide K step with the candidates as M (128 rows) and the H heads (padded
// to a multiple of 16) as N, so that each TMEM lane ends up holding one
// candidate's H head logits; the ReLU, the head weights and the head sum run
// in the epilogue on that one thread's registers.
//
// Candidates come in three forms:
//   kScoreBlocks  block representatives: pooled_hl rows (bf16 hi and lo of
//                 the fp32 mean, two accumulating UMMAs per K step);
//   kScoreFlat    every key s <= t (the flat scan);
//   kScoreHisa    the keys of the row's kept blocks (gathered block-wise by
//                 TMA: a kept block is one or more contiguous tile rows).
// e4m3 keys with d = 128 are multiplied on the fp8 tensor cores as loaded
// (kind::f8f6f4) against the query heads split into two e4m3 parts; e4m3 keys
// with d = 64 are staged as bytes and widened to bf16 in shared memory by
// four converter warps (exact).  Either way the per-token scale multiplies
// the finished score (ReLU(s*x) = s*ReLU(x) for s > 0).
//
// Work split: the (row, tile) pairs are laid out row-major with a fixed
// number of tile slots per row; CTA c takes the c-th contiguous range, so all
// SMs get equal shares whatever the number of rows.  Score keys go to a
// global row buffer that the selection kernel reads.
//
// Warp roles:
//   warp 0       TMA producer (keys / representatives, query heads)
//   warp 1       TMEM owner and UMMA issuer
//   warps 2-5    epilogue (TMEM -> registers -> score key -> global)
//   warps 6-9    e4m3 -> bf16 converters (e4m3 keys with d = 64 only)
// Every mbarrier wait is bounded; on expiry the CTA raises HISA_DEV_TIMEOUT,
// drains its outstanding copies and returns.
#include "hisa_pool.cuh"

namespace hisa {

namespace {

constexpr int kTileRows = 128;
constexpr int kHalfBytes = kTileRows * 128;   // one 128-byte-wide K slab of a tile
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpEpi0 = 2;
constexpr int kWarpConv0 = 6;
constexpr int kMinSmem = 120 * 1024;          // keeps one CTA (and its TMEM) per SM
constexpr int kMaxSmem = 232448;
constexpr int kSmem2 = 113 * 1024;            // per CTA when two share an SM
constexpr int kMinSmem2 = 80 * 1024;          // keeps it at two
constexpr int kMaxAcc = 4;
constexpr int kMaxStages = 8;
constexpr int kScaleRing = 16;                // e4m3 per-token scale slots (one tile each)
constexpr int kTabSubs = 256;                 // first key row of each sub-box, per row window

struct Layout {
    uint32_t a, s8, sc, tab, sel, q, w, bars, misc, total;
};

// Fused block selection scratch: the row's block score keys, a 256-bin
// histogram, scan / result words.
constexpr int kParentWords = kParentBits / 32;   // kept-superblock bitmap
constexpr int kSelScratch = kFuseMaxBlocks * 4 + 256 * 4 + 16 * 4 + kParentWords * 4;

// Accumulators of n columns that fit a CTA's share of TMEM's 512 columns (up to four).
__host__ __device__ inline int acc_count(int n, int per_sm) {
    const int c = 512 / per_sm / n;
    return c > 4 ? 4 : c;
}

// e4m3 keys with d = 128 are scored on the fp8 tensor cores directly (the
// 128-byte key rows are one swizzle row); d = 64 keys are widened to bf16.
__host__ __device__ constexpr bool uses_f8(int mode, bool e4m3, int d) {
    return e4m3 && d == 128 && mode != kScoreBlocks;
}

// Columns of one accumulator: the H heads (padded).  For fp8 scoring both
// e4m3 pieces of a query head accumulate into the head's column.
__host__ __device__ inline int acc_width(int mode, bool e4m3, int d, int npad) {
    (void)mode;
    (void)e4m3;
    (void)d;
    return npad;
}

__host__ __device__ constexpr int score_threads(int mode, bool e4m3, int d) {
    return e4m3 && !uses_f8(mode, e4m3, d) ? 320 : 192;
}

// Token and flat scoring of bf16 or fp8 keys run two CTAs per SM (half the
// shared memory and TMEM each) when the accumulators are at most 128 columns:
// two independent pipelines per SM hide each other's issue and drain gaps.
__host__ __device__ constexpr bool two_per_sm_kind(int mode, bool e4m3, int d) {
    return mode != kScoreBlocks && !(e4m3 && !uses_f8(mode, e4m3, d));
}


__host__ __device__ inline Layout score_layout(int mode, bool e4m3, int d, int npad, int sa, int s8) {
    const int halves = d / 64;
    const bool f8 = uses_f8(mode, e4m3, d);
    const int stage = f8 ? kTileRows * d : (mode == kScoreBlocks ? 2 : 1) * halves * kHalfBytes;
    Layout L;
    uint32_t off = 0;                        // from a 1024-byte aligned base
    L.a = off;
    off += sa * stage;
    L.s8 = off;
    off += e4m3 && !f8 ? s8 * kTileRows * d : 0;
    L.sc = off;
    off += (e4m3 && mode != kScoreBlocks) ? kScaleRing * kTileRows * 4 : 0;
    L.tab = off;
    off += kTabSubs * 4;
    L.sel = off;
    off += mode == kScoreBlocks ? kSelScratch : 0;
    off = (off + 1023u) & ~1023u;            // 128-byte-swizzled TMA boxes need 1024-byte alignment
    L.q = off;
    off += 2 * halves * npad * 128;
    L.w = off;
    off += 4 * 128 * 4;                      // one 128-float weight slot per epilogue warp
    L.bars = off;
    off += (4 * kMaxStages + 2 * kMaxAcc + 4 + 2 * kScaleRing) * 8;
    L.misc = off;
    off += 16;
    L.total = off;
    return L;
}

// Two CTAs per SM when the kind allows it, the accumulators fit half of TMEM
// and two operand stages fit half of the shared memory (wide heads at
// d = 128 do not: one CTA then takes the whole SM).
__host__ __device__ inline int ctas_per_sm(int mode, bool e4m3, int d, int npad) {
    if (!two_per_sm_kind(mode, e4m3, d) || acc_width(mode, e4m3, d, npad) > 128) return 1;
    return score_layout(mode, e4m3, d, npad, 2, 0).total + 1024 <= static_cast<uint32_t>(kSmem2) ? 2 : 1;
}

// TMEM allocation for `cols` accumulator columns: a power of two, at least 32.
__host__ __device__ inline uint32_t tmem_columns(int cols) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(cols)) c <<= 1;
    return c;
}

// Block scoring variants (a template parameter, so that each compiles alone):
// kBlocksAppend is the decode step (row b = sequence b, scored while the
// append kernel launched before it writes the new keys; see ScoreParams::app).
constexpr int kBlocksPlain = 0, kBlocksMasked = 1, kBlocksShard = 2, kBlocksAppend = 3, kBlocksGathered = 4;

// A query row: sequence, position, candidate slots, candidate tiles (0 if
// the row is invalid); app: the decode step appends a key at t first.
struct RowInfo {
    int b, t, lim, nt, app;
};

template <int MODE, int BV>
__device__ __forceinline__ RowInfo load_row(const ScoreParams& p, int row) {
    RowInfo R;
    R.lim = 0;
    R.nt = 0;
    R.app = 0;
    if (MODE == kScoreBlocks && BV == kBlocksAppend) {
        // decode step: the new key goes to position len[b] (nothing is
        // appended to a full sequence, whose last position is then cap - 1)
        R.b = row;
        const int n = p.len[row];
        if (n < 0 || n > p.cap) {
            R.t = -1;
            return R;
        }
        R.app = n < p.cap;
        R.t = R.app ? n : p.cap - 1;
        R.lim = R.t / p.B + 1;
    } else if (MODE == kScoreHisa) {
        const int4 pl = p.plan_in[row];     // written by the block selection
        R.b = pl.x;
        R.t = pl.y;
        if (R.t < 0) return R;
        R.lim = pl.z * p.B;                 // kept token slots
    } else if (MODE == kScoreBlocks && BV == kBlocksShard) {
        int own;
        const int vis = cp_visible_blocks(p.q_seq, p.q_pos, p.len, p.batch, p.cap, p.B, p.tok_off, row,
                                          &R.b, &own, &R.t);
        if (vis <= 0) {
            R.t = -1;
            return R;
        }
        R.lim = vis;                        // the shard's visible blocks
    } else {
        R.t = query_position(p.q_seq, p.q_pos, p.len, p.batch, p.cap, row, &R.b);
        if (R.t < 0) return R;
        R.lim = MODE == kScoreBlocks ? R.t / p.B + 1   // visible blocks
                                     : R.t + 1;        // visible keys
    }
    // the own block (the last visible one) is kept without a score: block
    // scoring covers blocks 0 .. lim - 2, in at least one tile (a shard need
    // not hold the own block: it scores all its visible blocks); gathered,
    // the row's slots are the children of its app = parent_n[row] kept
    // superblocks, bf per superblock
    int scored = (MODE == kScoreBlocks && BV != kBlocksShard) ? max(R.lim - 1, 1) : R.lim;
    if (MODE == kScoreBlocks && BV == kBlocksGathered) {
        R.app = min(max(p.parent_n[row], 0), p.parent_ld);
        scored = max(R.app * p.bf, 1);
    }
    R.nt = (scored + kTileRows - 1) / kTileRows;
    return R;
}

// Walks the row-major (row, tile) slots g0, g0 + 1, ... of a CTA's range
// without a 64-bit division per step.
struct TileCursor {
    long long g;
    int row, ti, tpr;
    __device__ __forceinline__ TileCursor(long long g0, int tiles_per_row)
        : g(g0), row(static_cast<int>(g0 / tiles_per_row)), ti(static_cast<int>(g0 % tiles_per_row)),
          tpr(tiles_per_row) {}
    __device__ __forceinline__ void next() {
        ++g;
        if (++ti == tpr) {
            ti = 0;
            ++row;
        }
    }
    __device__ __forceinline__ void next_row() {
        g += tpr - ti;
        ti = 0;
        ++row;
    }
};

// Position in a ring of n slots: slot and phase parity.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++slot == n) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t* status) {
    *abort_flag = 1;
    set_status(status, HISA_DEV_TIMEOUT);
}

// Lane 0 waits; the whole warp learns the outcome and is ordered after the
// wait (one waiting thread per warp keeps the barrier traffic off the shared
// memory pipe that the copies and the other roles need).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Eight e4m3 codes -> eight bf16 (exact: every e4m3 value is a bf16 value).
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 raw) {
    const uint32_t w[2] = {raw.x, raw.y};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const __nv_fp8x2_storage_t lo = static_cast<__nv_fp8x2_storage_t>(w[q] & 0xFFFFu);
        const __nv_fp8x2_storage_t hi = static_cast<__nv_fp8x2_storage_t>(w[q] >> 16);
        const float2 a = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(lo, __NV_E4M3)));
        const float2 b = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3)));
        o[2 * q] = pack_bf16x2(a.x, a.y);
        o[2 * q + 1] = pack_bf16x2(b.x, b.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// First key row of sub-box `sub` of tile `ti`.
template <int MODE>
__device__ __forceinline__ int tile_sub_row(const ScoreParams& p, const RowInfo& R, int row, int ti,
                                            int sub, int BR) {
    if (MODE == kScoreBlocks) return R.b * p.nblk + ti * kTileRows;
    if (MODE == kScoreFlat) return R.b * p.cap + ti * kTileRows + sub * BR;
    const int slot = ti * kTileRows + sub * BR;
    const int blk = slot < R.lim ? __ldg(p.blocks + static_cast<size_t>(row) * p.mm + slot / p.B) : 0;
    return R.b * p.cap + blk * p.B + slot % p.B;
}

// Shared-memory load the compiler keeps in place (the head weights are read
// per tile instead of being held in registers across the tile loop).
__device__ __forceinline__ float4 lds_f32x4(const float* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}

// sum_h w_h * ReLU(acc_h) over the npad head columns of one TMEM lane, 16
// columns (one TMEM load) at a time in a loop that is not unrolled: the code
// stays a few cache lines, which is what the first tile after a cold start
// waits for; four interleaved partial sums (fixed order: a[j] adds heads
// j, j + 4, ... in turn).
__device__ __forceinline__ float head_sum(int npad, uint32_t taddr, const float* wv) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int g = 0; g < npad; g += 16) {
        uint32_t r[16];
        tmem_ld16_nowait(taddr + g, r);
        // the group's head weights load while the TMEM load is in flight
        float4 wg[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) wg[q] = lds_f32x4(wv + g + 4 * q);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            fma2(a[0], a[1], wg[q].x, wg[q].y, fmaxf(__uint_as_float(r[4 * q]), 0.f),
                 fmaxf(__uint_as_float(r[4 * q + 1]), 0.f));
            fma2(a[2], a[3], wg[q].z, wg[q].w, fmaxf(__uint_as_float(r[4 * q + 2]), 0.f),
                 fmaxf(__uint_as_float(r[4 * q + 3]), 0.f));
        }
    }
    return (a[0] + a[1]) + (a[2] + a[3]);
}

// ---------------------------------------------- fused block selection
// Run by the four epilogue warps (thread e = 0..127) on one row's block score
// keys in shared memory; the same rule as the selection kernel: the top kk
// keys, ties to the lower slot, kept slots in ascending order.

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Exclusive scan of one value per epilogue thread (in thread order).
__device__ __forceinline__ uint32_t epi_scan(uint32_t v, int e, uint32_t* misc) {
    const int w = e >> 5, l = e & 31;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (l >= o) incl += x;
    }
    if (l == 31) misc[w] = incl;
    epi_bar();
    uint32_t before = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) before += i < w ? misc[i] : 0u;
    epi_bar();
    return before + incl - v;
}

// The kk-th largest of the keys s[0..n) (0 < kk < their count; with MASKED,
// key 0 marks a masked slot and is not counted): four 8-bit radix rounds from
// the top.  Returns T; *take_eq = how many keys equal to T are among the top kk.
template <bool MASKED>
__device__ uint32_t epi_threshold(const uint32_t* s, int n, int kk, uint32_t* hist, uint32_t* misc, int e,
                                  int* take_eq) {
    uint32_t prefix = 0, mask = 0;
    uint32_t krem = static_cast<uint32_t>(kk);
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[e] = 0;
        hist[e + 128] = 0;
        epi_bar();
        for (int c = e; c < n; c += 128) {
            const uint32_t x = s[c];
            if ((!MASKED || x != 0u) && (x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
        }
        epi_bar();
        // thread e owns bins 255 - 2e and 254 - 2e (highest first)
        const uint32_t h0 = hist[255 - 2 * e], h1 = hist[254 - 2 * e];
        const uint32_t excl = epi_scan(h0 + h1, e, misc);
        if (excl < krem && krem <= excl + h0 + h1) {
            const bool first = krem <= excl + h0;
            misc[4] = static_cast<uint32_t>(first ? 255 - 2 * e : 254 - 2 * e);
            misc[5] = first ? krem - excl : krem - excl - h0;
        }
        epi_bar();
        prefix |= misc[4] << shift;
        mask |= 255u << shift;
        krem = misc[5];
        epi_bar();
    }
    *take_eq = static_cast<int>(krem);
    return prefix;
}

// Writes the slots of the keys of s[0..n) above T, plus the first take_eq
// equal to T, in ascending order to out (and dbg); with par, slot c is
// written as block par[c / bf] * bf + c % bf.
__device__ __noinline__ void epi_emit(const uint32_t* s, int n, uint32_t T, int take_eq, int32_t* out,
                                      int32_t* dbg, uint32_t* misc, int e, const int32_t* par = nullptr,
                                      int bf = 1) {
    const int w = e >> 5, l = e & 31;
    const int per = ((n + 3) / 4 + 31) & ~31;
    const int w0 = w * per;
    const int w1 = min(n, w0 + per);
    uint32_t gt = 0, eq = 0;
    for (int base = w0; base < w1; base += 32) {
        const int c = base + l;
        const uint32_t x = c < w1 ? s[c] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, c < w1 && x > T));
        eq += __popc(__ballot_sync(0xffffffffu, c < w1 && x == T));
    }
    if (l == 0) {
        misc[8 + w] = gt;
        misc[12 + w] = eq;
    }
    epi_bar();
    uint32_t eq_run = 0, pos = 0;
    {
        uint32_t eqb = 0, off = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t ei = misc[12 + i];
            const int room = take_eq - static_cast<int>(eqb);
            const uint32_t take = room <= 0 ? 0u : (static_cast<uint32_t>(room) < ei ? room : ei);
            if (i == w) {
                eq_run = eqb;
                pos = off;
            }
            eqb += ei;
            off += misc[8 + i] + take;
        }
    }
    const unsigned lt = (1u << l) - 1u;
    for (int base = w0; base < w1; base += 32) {
        const int c = base + l;
        const uint32_t x = c < w1 ? s[c] : 0u;
        const bool is_gt = c < w1 && x > T;
        const bool is_eq = c < w1 && x == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t eq_rank = eq_run + __popc(eqm & lt);
        const bool sel = is_gt || (is_eq && eq_rank < static_cast<uint32_t>(take_eq));
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const int at = static_cast<int>(pos + __popc(selm & lt));
            const int id = par ? par[c / bf] * bf + c % bf : c;
            out[at] = id;
            if (dbg) dbg[at] = id;
        }
        eq_run += __popc(eqm);
        pos += __popc(selm);
    }
}


// BV (block scoring only): every visible block is a candidate (kBlocksPlain),
// a kept-superblock list masks the blocks outside it (kBlocksMasked), only
// the children of the kept superblocks are loaded and scored, bf at a time,
// slot q * bf + c being child c of the q-th kept superblock (kBlocksGathered),
// or the cache is a context-parallel shard (kBlocksShard).
template <int MODE, bool E4M3, int D, int BV>
__global__ void __launch_bounds__(score_threads(MODE, E4M3, D), two_per_sm_kind(MODE, E4M3, D) ? 2 : 1)
    score_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap qmap,
                 const ScoreParams p) {
    constexpr int kHalves = D / 64;
    constexpr int kOps = (MODE == kScoreBlocks) ? 2 : 1;
    constexpr bool kF8 = uses_f8(MODE, E4M3, D);          // fp8 operands straight from TMA
    constexpr bool kConv = E4M3 && !kF8;                  // e4m3 widened to bf16 by converter warps
    constexpr bool PAR = MODE == kScoreBlocks && BV == kBlocksMasked;
    constexpr bool GAT = MODE == kScoreBlocks && BV == kBlocksGathered;
    constexpr bool APP = MODE == kScoreBlocks && BV == kBlocksAppend;
    constexpr int kStageBytes = kF8 ? kTileRows * D : kOps * kHalves * kHalfBytes;
    constexpr int kStage8Bytes = kTileRows * D;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int SA = p.stages;                    // bf16 operand stages
    const int S8 = kConv ? p.stages8 : 1;       // e4m3 staging stages
    const Layout L = score_layout(MODE, E4M3, D, p.npad, SA, S8);
    const int NW = acc_width(MODE, E4M3, D, p.npad);   // accumulator columns
    const int NACC = p.nacc;
    uint8_t* sA = smem + L.a;
    uint8_t* s8 = smem + L.s8;
    uint8_t* sQ = smem + L.q;
    float* sS = reinterpret_cast<float*>(smem + L.sc);   // e4m3 scales [kScaleRing][128]
    float* sW = reinterpret_cast<float*>(smem + L.w);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* full = bars;                         // operand stage ready   [SA]
    uint64_t* empty = bars + kMaxStages;           // operand stage free    [SA]
    uint64_t* sfull = bars + 2 * kMaxStages;       // e4m3 staging landed   [S8]
    uint64_t* sempty = bars + 3 * kMaxStages;      // e4m3 staging consumed [S8]
    uint64_t* tfull = bars + 4 * kMaxStages;       // accumulator ready   [kMaxAcc]
    uint64_t* tempty = tfull + kMaxAcc;            // accumulator drained [kMaxAcc]
    uint64_t* qfull = tempty + kMaxAcc;            // query heads landed  [2]
    uint64_t* qempty = qfull + 2;                  // query heads free    [2]
    uint64_t* scfull = qempty + 2;                 // tile scales landed  [kScaleRing]
    uint64_t* scempty = scfull + kScaleRing;       // tile scales read    [kScaleRing]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int npad = p.npad;
    const uint32_t ncols = tmem_columns(NACC * NW);
    const int q_slot_bytes = kHalves * npad * 128;
    const int tpr = p.tiles_per_row;
    const int BR = (MODE == kScoreBlocks) ? kTileRows : (p.B < kTileRows ? p.B : kTileRows);
    const int nsub = kTileRows / BR;
    // contiguous ranges of (row, tile) slots; whole rows when the block
    // selection is fused in
    const bool fuse = MODE == kScoreBlocks && p.fuse && tpr * kTileRows <= kFuseMaxBlocks;
    const long long g0 = fuse ? static_cast<long long>(p.n_q) * blockIdx.x / gridDim.x * tpr
                              : p.total_tiles * blockIdx.x / gridDim.x;
    const long long g1 = fuse ? static_cast<long long>(p.n_q) * (blockIdx.x + 1) / gridDim.x * tpr
                              : p.total_tiles * (blockIdx.x + 1) / gridDim.x;

    if (warp == kWarpProducer && lane == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(full + s, kConv ? 4 : 1);
            mbar_init(empty + s, 1);
        }
        for (int s = 0; s < S8; ++s) {
            mbar_init(sfull + s, 1);
            mbar_init(sempty + s, 4);
        }
        for (int a = 0; a < kMaxAcc; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 4);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(qfull + a, 1);
            mbar_init(qempty + a, 1);
        }
        for (int r = 0; r < kScaleRing; ++r) {
            mbar_init(scfull + r, kConv ? 32 : 1);   // per producer lane (converter path) or lane 0
            mbar_init(scempty + r, 4);     // one per epilogue warp
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_async_smem();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&qmap);
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // everything above overlaps the previous kernel; its outputs are read
    // below.  In the decode step the previous kernel is the append, which this
    // kernel does not wait for here (see ScoreParams::app).
    if (!APP) grid_dependency_wait();
    grid_launch_dependents();

    if (warp == kWarpProducer) {
        // keys read by one row only stream through L2; keys that several rows
        // read (a prefill chunk) stay
        const uint64_t pol = p.keep_keys ? policy_evict_last() : policy_evict_first();
        const long long key_rows = static_cast<long long>(p.batch) * p.cap;
        int it = 0, qloads = 0, cur_row = -1, tb = 0;
        RowInfo R;
        R.nt = 0;
        int win_cur = 0, win_nxt = 0, cur_w = 0;
        bool ok = true;
        const int NS = kConv ? S8 : SA;
        Ring ring;
        if constexpr (!kConv) {
            // bf16 and fp8 keys: per row, the warp stages the sub-boxes' first
            // key rows in shared memory; lane 0 alone then issues the row's
            // tiles, one barrier wait and one transaction count per tile
            int* sTab = reinterpret_cast<int*>(smem + L.tab);
            TileCursor cur(g0, tpr);
            while (cur.g < g1 && ok) {
                const int row = cur.row;
                // kept-block ids of the row's first window, loaded together
                // with the row's plan rather than after it (one L2 round trip
                // per row start instead of two); the ids are read within the
                // row's [0, mm) entries and only used where the plan says so
                constexpr int kPre = kTabSubs / 32;
                int pre[kPre];
                if constexpr (MODE == kScoreHisa) {
                    const int32_t* brow = p.blocks + static_cast<size_t>(row) * p.mm;
                    const int wmax = min(tpr - cur.ti, kTabSubs / nsub) * nsub;
#pragma unroll
                    for (int q = 0; q < kPre; ++q) {
                        const int j = lane + 32 * q;
                        const int slot = (cur.ti + j / nsub) * kTileRows + (j % nsub) * BR;
                        pre[q] = j < wmax ? __ldg(brow + min(slot / p.B, p.mm - 1)) : 0;
                    }
                }
                R = load_row<MODE, BV>(p, row);
                const long long left = g1 - cur.g;
                const int t_end = static_cast<int>(R.nt < cur.ti + left ? R.nt : cur.ti + left);
                if (cur.ti >= t_end) {
                    cur.next_row();
                    continue;
                }
                if constexpr (GAT) {
                    // the row's kept superblocks, for lane 0's boxes
                    for (int i = lane; i < R.app; i += 32)
                        sTab[i] = p.parent[static_cast<size_t>(row) * p.parent_ld + i];
                    __syncwarp();
                }
                const int qs = qloads & 1;
                if (qloads >= 2 && !warp_wait(qempty + qs, ((qloads - 2) >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(qfull + qs, q_slot_bytes);
                    if (kF8) {
                        // the row's split heads: one [2 npad x 128 B] box
                        tma_load_2d(sQ + qs * q_slot_bytes, &qmap, qfull + qs, 0, row * 2 * npad);
                    } else {
#pragma unroll
                        for (int kh = 0; kh < kHalves; ++kh)
                            tma_load_2d(sQ + qs * q_slot_bytes + kh * npad * 128, &qmap, qfull + qs, kh * 64,
                                        row * p.H);
                    }
                }
                ++qloads;
                for (int t = cur.ti; t < t_end && ok;) {
                    const int nwin = min(t_end - t, kTabSubs / nsub);
                    if (MODE == kScoreHisa) {
                        if (t == cur.ti) {
#pragma unroll
                            for (int q = 0; q < kPre; ++q) {
                                const int j = lane + 32 * q;
                                if (j < nwin * nsub) {
                                    const int slot = (t + j / nsub) * kTileRows + (j % nsub) * BR;
                                    sTab[j] = R.b * p.cap + (slot < R.lim ? pre[q] : 0) * p.B + slot % p.B;
                                }
                            }
                        } else {
                            for (int j = lane; j < nwin * nsub; j += 32)
                                sTab[j] = tile_sub_row<MODE>(p, R, row, t + j / nsub, j % nsub, BR);
                        }
                        __syncwarp();
                    }
                    if (lane == 0) {
                        for (int k = 0; k < nwin; ++k) {
                            if (!mbar_wait(empty + ring.slot, ring.phase ^ 1u, abort_flag) ||
                                (kF8 && !mbar_wait(scempty + (it & (kScaleRing - 1)),
                                                   ((it / kScaleRing) & 1) ^ 1, abort_flag))) {
                                ok = false;
                                break;
                            }

                            uint64_t* fb = full + ring.slot;
                            uint8_t* dst = sA + ring.slot * kStageBytes;
                            if (GAT) {
                                // one run of bf representatives per kept superblock of the
                                // tile (boxes of bf rows; runs past the list are not loaded
                                // and their slots are masked)
                                const int runs = kTileRows / p.bf;
                                const int q0 = (t + k) * runs;
                                const int nr = max(0, min(runs, R.app - q0));
                                mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nr * p.bf * 2 * kHalves * 128));
                                for (int r = 0; r < nr; ++r)
#pragma unroll 1
                                    for (int h = 0; h < 2 * kHalves; ++h)
                                        tma_load_3d(dst + h * kHalfBytes + r * p.bf * 128, &amap, fb,
                                                    (h / kHalves) * D + (h % kHalves) * 64, sTab[q0 + r] * p.bf,
                                                    R.b);
                            } else if (MODE == kScoreBlocks) {
                                // [batch, nblk, 2d] boxes: the rows past the sequence's
                                // blocks are zero-filled, not read
                                mbar_arrive_expect_tx(fb, kStageBytes);
#pragma unroll
                                for (int op = 0; op < 2; ++op)
#pragma unroll
                                    for (int kh = 0; kh < kHalves; ++kh)
                                        tma_load_3d(dst + (op * kHalves + kh) * kHalfBytes, &amap, fb,
                                                    op * D + kh * 64, (t + k) * kTileRows, R.b);
                            } else {
                                mbar_arrive_expect_tx(fb, kStageBytes);
                                for (int sub = 0; sub < nsub; ++sub) {
                                    const int srow = MODE == kScoreHisa
                                                         ? sTab[k * nsub + sub]
                                                         : R.b * p.cap + (t + k) * kTileRows + sub * BR;
                                    if (kF8) {
                                        tma_load_2d_hint(dst + sub * BR * D, &amap, fb, 0, srow, pol);
                                    } else {
#pragma unroll
                                        for (int kh = 0; kh < kHalves; ++kh)
                                            tma_load_2d_hint(dst + kh * kHalfBytes + sub * BR * 128, &amap, fb,
                                                             kh * 64, srow, pol);
                                    }
                                }
                            }
                            if (kF8) {
                                // the tile's per-token scales into the scale ring
                                const int sc = it & (kScaleRing - 1);   // free: waited above
                                float* sdst = sS + sc * kTileRows;
                                if (p.scale_bulk) {
                                    uint32_t bytes = 0;
                                    for (int sub = 0; sub < nsub; ++sub) {
                                        const long long srow = MODE == kScoreHisa
                                                                   ? sTab[k * nsub + sub]
                                                                   : R.b * p.cap + (t + k) * kTileRows + sub * BR;
                                        const long long nv = key_rows - srow < BR ? key_rows - srow : BR;
                                        bytes += nv > 0 ? static_cast<uint32_t>(nv) * 4u : 0u;
                                    }
                                    mbar_arrive_expect_tx(scfull + sc, bytes);
                                    for (int sub = 0; sub < nsub; ++sub) {
                                        const long long srow = MODE == kScoreHisa
                                                                   ? sTab[k * nsub + sub]
                                                                   : R.b * p.cap + (t + k) * kTileRows + sub * BR;
                                        const long long nv = key_rows - srow < BR ? key_rows - srow : BR;
                                        if (nv > 0)
                                            bulk_load(sdst + sub * BR, p.key_scale + srow,
                                                      static_cast<uint32_t>(nv) * 4u, scfull + sc);
                                    }
                                } else {
                                    for (int r = 0; r < kTileRows; ++r) {
                                        const int sub = r / BR;
                                        const long long srow =
                                            (MODE == kScoreHisa ? sTab[k * nsub + sub]
                                                                : R.b * p.cap + (t + k) * kTileRows + sub * BR) +
                                            (r - sub * BR);
                                        if (srow < key_rows) cp_async_4(sdst + r, p.key_scale + srow);
                                    }
                                    cp_async_arrive_noinc(scfull + sc);
                                }
                            }
                            ++it;
                            ring.next(SA);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    it = __shfl_sync(0xffffffffu, it, 0);
                    ring.slot = __shfl_sync(0xffffffffu, ring.slot, 0);
                    ring.phase = __shfl_sync(0xffffffffu, ring.phase, 0);
                    __syncwarp();
                    t += nwin;
                }
                if (t_end < R.nt) break;   // the range ends inside this row
                cur.next_row();
            }
        } else
        for (TileCursor cur(g0, tpr); cur.g < g1 && ok;) {
            const int row = cur.row;
            const int ti = cur.ti;
            if (row != cur_row) {
                cur_row = row;
                R = load_row<MODE, BV>(p, row);
                if (ti < R.nt) {
                    // new row with work here: its query heads and block-id windows
                    const int qs = qloads & 1;
                    if (qloads >= 2 && !warp_wait(qempty + qs, ((qloads - 2) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(qfull + qs, q_slot_bytes);
#pragma unroll
                        for (int kh = 0; kh < kHalves; ++kh)
                            tma_load_2d(sQ + qs * q_slot_bytes + kh * npad * 128, &qmap, qfull + qs,
                                        kh * 64, row * p.H);
                    }
                    ++qloads;
                    tb = ti;
                    const int nsub_row = (R.nt - tb) * nsub;
                    const int gsub0 = lane, gsub1 = 32 + lane;
                    win_cur = gsub0 < nsub_row
                                  ? tile_sub_row<MODE>(p, R, row, tb + gsub0 / nsub, gsub0 % nsub, BR)
                                  : 0;
                    win_nxt = gsub1 < nsub_row
                                  ? tile_sub_row<MODE>(p, R, row, tb + gsub1 / nsub, gsub1 % nsub, BR)
                                  : 0;
                    cur_w = 0;
                }
            }
            if (ti >= R.nt) {
                cur.next_row();
                continue;
            }
            const int gs = (ti - tb) * nsub;
            if ((gs >> 5) != cur_w) {
                cur_w = gs >> 5;
                win_cur = win_nxt;
                const int gn = 32 * (cur_w + 1) + lane;
                win_nxt = gn < (R.nt - tb) * nsub
                              ? tile_sub_row<MODE>(p, R, row, tb + gn / nsub, gn % nsub, BR)
                              : 0;
            }
            const int ss = ring.slot;
            const uint32_t ph = ring.phase;
            uint64_t* fb = E4M3 ? sfull + ss : full + ss;
            uint64_t* eb = E4M3 ? sempty + ss : empty + ss;
            if (!warp_wait(eb, ph ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            if (MODE == kScoreBlocks) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, kStageBytes);
#pragma unroll
                    for (int op = 0; op < 2; ++op)
#pragma unroll
                        for (int kh = 0; kh < kHalves; ++kh)
                            tma_load_3d(sA + ss * kStageBytes + (op * kHalves + kh) * kHalfBytes, &amap, fb,
                                        op * D + kh * 64, ti * kTileRows, R.b);
                }
            } else {
                if (lane == 0) mbar_arrive_expect_tx(fb, E4M3 ? kStage8Bytes : kStageBytes);
                for (int sub = 0; sub < nsub; ++sub) {
                    const int srow = __shfl_sync(0xffffffffu, win_cur, (gs & 31) + sub);
                    if (lane != 0) continue;
                    if (E4M3) {
                        tma_load_2d_hint(s8 + ss * kStage8Bytes + sub * BR * D, &amap, fb, 0, srow, pol);
                    } else {
#pragma unroll
                        for (int kh = 0; kh < kHalves; ++kh)
                            tma_load_2d_hint(sA + ss * kStageBytes + kh * kHalfBytes + sub * BR * 128, &amap,
                                             fb, kh * 64, srow, pol);
                    }
                }
            }
            if (E4M3) {
                // the tile's per-token scales, one 4-byte copy per key row
                const int sc = it & (kScaleRing - 1);
                if (!warp_wait(scempty + sc, ((it / kScaleRing) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int q = 0; q < kTileRows / 32; ++q) {
                    const int r = q * 32 + lane;
                    const int sub = r / BR;
                    int srow = __shfl_sync(0xffffffffu, win_cur, (gs & 31) + (sub < nsub ? sub : 0));
                    srow = MODE == kScoreFlat ? R.b * p.cap + ti * kTileRows + r : srow + (r - sub * BR);
                    if (srow < key_rows) cp_async_4(sS + sc * kTileRows + r, p.key_scale + srow);
                }
                cp_async_arrive_noinc(scfull + sc);
            }
            __syncwarp();
            ++it;
            ring.next(NS);
            cur.next();
        }
        if (E4M3) cp_async_wait_all();   // no scale copy still landing at exit
        if (lane == 0) {
            if (!ok) raise_abort(abort_flag, p.status);
            if (kF8 && !ok)
                for (int n = it > kScaleRing ? it - kScaleRing : 0; n < it; ++n)
                    mbar_wait(scfull + (n & (kScaleRing - 1)), (n / kScaleRing) & 1, nullptr);
            // Drain: no copy into, and no arrive on, this CTA's shared memory
            // may still be pending when it exits.
            for (int n = it > NS ? it - NS : 0; n < it; ++n) {
                const int s = n % NS;
                const uint32_t ph = (n / NS) & 1;
                if (ok) mbar_wait(kConv ? sempty + s : empty + s, ph, nullptr);
                else mbar_wait(kConv ? sfull + s : full + s, ph, nullptr);
            }
            if (qloads >= 1) {
                if (ok && qloads >= 2)
                    mbar_wait(qempty + ((qloads - 2) & 1), ((qloads - 2) >> 1) & 1, nullptr);
                if (!ok) mbar_wait(qfull + ((qloads - 1) & 1), ((qloads - 1) >> 1) & 1, nullptr);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = kF8 ? idesc_e4m3_f32(static_cast<uint32_t>(npad))
                                       : idesc_bf16_f32(static_cast<uint32_t>(npad));
            int it = 0, qloads = 0, cur_row = -1;
            uint32_t q_base = 0;
            RowInfo R;
            R.nt = 0;
            bool ok = true;
            Ring rs, ra;   // operand stage, accumulator
            for (TileCursor cur(g0, tpr); cur.g < g1 && ok;) {
                const int row = cur.row;
                const int ti = cur.ti;
                if (row != cur_row) {
                    cur_row = row;
                    R = load_row<MODE, BV>(p, row);
                    if (ti < R.nt) {
                        if (qloads > 0) umma_commit(qempty + ((qloads - 1) & 1));
                        if (!mbar_wait(qfull + (qloads & 1), (qloads >> 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        q_base = smem_addr(sQ + (qloads & 1) * q_slot_bytes);
                        ++qloads;
                    }
                }
                if (ti >= R.nt) {
                    cur.next_row();
                    continue;
                }
                const int s = rs.slot;
                const int a = ra.slot;
                if (!mbar_wait(full + s, rs.phase, abort_flag) ||
                    !mbar_wait(tempty + a, ra.phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * NW);
                const uint32_t a_base = smem_addr(sA + s * kStageBytes);
                // (loops kept rolled: a few instructions of code for the cold start)
                if (kF8) {
                    // 128 candidates x npad heads x 128 bytes: four K = 32 steps,
                    // each for the q1 piece and then the q2 piece of every head
                    // (rows npad .. 2 npad - 1 of the split heads) into the same
                    // accumulator: D = K (q1 + q2)^T
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = sw128_kmajor_desc(a_base + kk * 32);
                        umma_e4m3(d_tmem, adesc, sw128_kmajor_desc(q_base + kk * 32), idesc, kk ? 1u : 0u);
                        umma_e4m3(d_tmem, adesc, sw128_kmajor_desc(q_base + npad * 128 + kk * 32), idesc, 1u);
                    }
                } else {
#pragma unroll 1
                    for (int k = 0; k < kHalves * 4; ++k) {
                        const int kh = k >> 2, kk = k & 3;
                        const uint64_t bdesc = sw128_kmajor_desc(q_base + kh * npad * 128 + kk * 32);
                        const uint64_t adesc = sw128_kmajor_desc(a_base + kh * kHalfBytes + kk * 32);
                        umma_bf16(d_tmem, adesc, bdesc, idesc, k ? 1u : 0u);
                        if (MODE == kScoreBlocks) {
                            const uint64_t ldesc =
                                sw128_kmajor_desc(a_base + (kHalves + kh) * kHalfBytes + kk * 32);
                            umma_bf16(d_tmem, ldesc, bdesc, idesc, 1u);
                        }
                    }
                }
                umma_commit(empty + s);
                umma_commit(tfull + a);
                ++it;
                rs.next(SA);
                ra.next(NACC);
                cur.next();
            }
            if (!ok) raise_abort(abort_flag, p.status);
            // every UMMA of this CTA has finished before TMEM is released
            if (it > 0) mbar_wait(tfull + ((it - 1) % NACC), ((it - 1) / NACC) & 1, nullptr);
        }
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
        const int quad = warp & 3;                    // TMEM lanes this warp may read
        const int r = quad * 32 + lane;               // tile row = candidate
        float* wv = sW + (warp - kWarpEpi0) * 128;
        const int e = (warp - kWarpEpi0) * 32 + lane;                 // 0..127
        uint32_t* sKeys = reinterpret_cast<uint32_t*>(smem + L.sel);  // fused selection
        uint32_t* sHist = sKeys + kFuseMaxBlocks;
        uint32_t* sMisc = sHist + 256;
        uint32_t* sPar = sMisc + 16;                                   // kept superblocks (bits)
        int it = 0, cur_row = -1;
        RowInfo R;
        R.nt = 0;
        int own0 = 0, own_t = 0;     // first slot of the own block (listed last), t within it
        bool ok = true;
        Ring ra;
        for (TileCursor cur(g0, tpr); cur.g < g1;) {
            const int row = cur.row;
            const int ti = cur.ti;
            if (row != cur_row) {
                cur_row = row;
                R = load_row<MODE, BV>(p, row);
                if (MODE == kScoreHisa && R.nt > 0) {
                    own0 = R.lim - p.B;
                    own_t = R.t % p.B;
                }
                if (fuse && R.nt == 0) {
                    // query position outside its sequence: no blocks
                    int32_t* bl = p.sel_blocks + static_cast<size_t>(row) * p.mm;
                    int32_t* bd = p.sel_blocks_out ? p.sel_blocks_out + static_cast<size_t>(row) * p.mm : nullptr;
                    for (int i = e; i < p.mm; i += 128) {
                        bl[i] = -1;
                        if (bd) bd[i] = -1;
                    }
                    if (e == 0) {
                        p.sel_nblocks[row] = 0;
                        if (p.sel_nblocks_out) p.sel_nblocks_out[row] = 0;
                        p.sel_plan[row] = make_int4(R.b, -1, 0, 0);
                        set_status(p.status, HISA_DEV_BAD_QUERY);
                    }
                }
                if (GAT && ti < R.nt) {
                    // the row's kept superblocks (slot q * bf + c: child c of the q-th)
                    epi_bar();
                    for (int i = e; i < R.app; i += 128)
                        reinterpret_cast<int32_t*>(sPar)[i] = p.parent[static_cast<size_t>(row) * p.parent_ld + i];
                    epi_bar();
                }
                if (MODE == kScoreBlocks && PAR && ti < R.nt) {
                    // the row's kept superblocks as a bitmap
                    epi_bar();
                    const int nwords = ((R.lim - 1) / p.bf) / 32 + 1;
                    for (int i = e; i < nwords; i += 128) sPar[i] = 0u;
                    epi_bar();
                    for (int i = e; i < p.parent_ld; i += 128) {
                        const int v = p.parent[static_cast<size_t>(row) * p.parent_ld + i];
                        if (v >= 0 && v < nwords * 32) atomicOr(&sPar[v >> 5], 1u << (v & 31));
                    }
                    epi_bar();
                }
                if (ti < R.nt) {
                    __syncwarp();
                    for (int h = lane; h < 128; h += 32)
                        wv[h] = kF8 ? (h < npad ? p.w8[static_cast<size_t>(row) * npad + h] : 0.f)
                                    : (h < p.H ? p.w[row * p.H + h] : 0.f);
                    __syncwarp();
                }
            }
            if (ti >= R.nt) {
                cur.next_row();
                continue;
            }
            const int c = ti * kTileRows + r;
            bool valid;
            if (MODE == kScoreBlocks) {
                valid = c < (BV == kBlocksShard ? R.lim : R.lim - 1);   // the candidates
                if (GAT) {
                    const int q = c / p.bf;
                    valid = q < R.app && reinterpret_cast<const int32_t*>(sPar)[q] * p.bf + (c - q * p.bf) < R.lim - 1;
                }
                if (PAR && valid) {
                    const int sb = c / p.bf;
                    valid = (sPar[sb >> 5] >> (sb & 31)) & 1u;
                }
            } else if (MODE == kScoreFlat) {
                valid = c <= R.t;
            } else {
                valid = c < own0 || (c < R.lim && c - own0 <= own_t);
            }
            const int a = ra.slot;
            float acc = 0.f;
            if (ok && warp_wait(tfull + a, ra.phase, abort_flag)) {
                tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                       static_cast<uint32_t>(a * NW);
                acc = head_sum(npad, taddr, wv);
                tc_fence_before();
            } else if (ok) {
                ok = false;
                raise_abort(abort_flag, p.status);
            }
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive(tempty + a);
            if (E4M3) {
                const int sc = it & (kScaleRing - 1);
                float scale = 1.f;
                if (ok && warp_wait(scfull + sc, (it / kScaleRing) & 1, abort_flag)) {
                    scale = sS[sc * kTileRows + r];
                } else if (ok) {
                    ok = false;
                    raise_abort(abort_flag, p.status);
                }
                __syncwarp();
                if (lane == 0 && ok) mbar_arrive(scempty + sc);
                acc *= scale;
            }
            if (fuse) sKeys[c] = valid ? score_key(acc) : 0u;
            else p.out[static_cast<size_t>(row) * p.ldo + c] = valid ? score_key(acc) : 0u;
            if (p.counts) {
                const bool slot = MODE == kScoreBlocks ? valid : c < R.lim;
                // the own block counts as a visible block once per row
                const int own = MODE == kScoreBlocks && BV != kBlocksShard && ti == 0 && e == 0;
                const int n = __popc(__ballot_sync(0xffffffffu, slot)) + own;
                if (lane == 0 && n)
                    atomicAdd(p.counts + static_cast<size_t>(row) * p.counts_ld + p.counts_col +
                                  (MODE == kScoreBlocks ? 0 : 1),
                              static_cast<unsigned long long>(n));
            }
            if (fuse && ti == R.nt - 1) {
                // the row is scored: keep its own block and the best m - 1 others
                epi_bar();
                const int nb = R.lim;                  // visible blocks; the own block is nb - 1
                int32_t* bl = p.sel_blocks + static_cast<size_t>(row) * p.mm;
                int32_t* bd = p.sel_blocks_out ? p.sel_blocks_out + static_cast<size_t>(row) * p.mm : nullptr;
                // candidates: the nonzero keys of blocks 0 .. nb - 2 (a kept-superblock
                // list masks the others to 0), or of the gathered slots
                const int nsl = GAT ? R.app * p.bf : nb - 1;
                const int32_t* par = GAT ? reinterpret_cast<const int32_t*>(sPar) : nullptr;
                uint32_t nv = static_cast<uint32_t>(nsl);
                if (PAR || GAT) {
                    nv = 0;
                    for (int c = e; c < nsl; c += 128) nv += sKeys[c] != 0u;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
                    if (lane == 0) sMisc[12 + (e >> 5)] = nv;
                    epi_bar();
                    nv = sMisc[12] + sMisc[13] + sMisc[14] + sMisc[15];
                    epi_bar();
                }
                const int kk = p.m - 1;
                const int kept = static_cast<int>(nv) <= kk ? static_cast<int>(nv) : kk;
                if (static_cast<int>(nv) <= kk) {
                    if (PAR || GAT) {
                        if (nv > 0) epi_emit(sKeys, nsl, 0u, 0, bl, bd, sMisc, e, par, p.bf);   // every unmasked one
                    } else {
                        for (int i = e; i < kept; i += 128) {                         // every candidate
                            bl[i] = i;
                            if (bd) bd[i] = i;
                        }
                    }
                } else if (kk > 0) {
                    int take_eq;
                    const uint32_t T = epi_threshold<PAR || GAT>(sKeys, nsl, kk, sHist, sMisc, e, &take_eq);
                    epi_emit(sKeys, nsl, T, take_eq, bl, bd, sMisc, e, par, p.bf);
                }
                for (int i = kept + e; i < p.mm; i += 128) {
                    const int v = i == kept ? nb - 1 : -1;   // own block last
                    bl[i] = v;
                    if (bd) bd[i] = v;
                }
                const int keep = kept + 1;
                if (e == 0) {
                    p.sel_nblocks[row] = keep;
                    if (p.sel_nblocks_out) p.sel_nblocks_out[row] = keep;
                    p.sel_plan[row] = make_int4(R.b, R.t, keep, 0);
                    if (APP && R.app) {
                        grid_dependency_wait();    // the append kernel has finished
                        p.len_w[R.b] = R.t + 1;
                    }
                }
                epi_bar();
            }
            ++it;
            ra.next(NACC);
            cur.next();
        }
    } else if (kConv && warp >= kWarpConv0) {
        const int cw = warp - kWarpConv0;
        int it = 0, cur_row = -1;
        RowInfo R;
        R.nt = 0;
        bool ok = true;
        Ring r8, rs;   // staging slot, operand stage
        for (TileCursor cur(g0, tpr); cur.g < g1 && ok;) {
            const int row = cur.row;
            const int ti = cur.ti;
            if (row != cur_row) {
                cur_row = row;
                R = load_row<MODE, BV>(p, row);
            }
            if (ti >= R.nt) {
                cur.next_row();
                continue;
            }
            const int s8i = r8.slot;
            const int sa = rs.slot;
            if (!warp_wait(sfull + s8i, r8.phase, abort_flag) ||
                !warp_wait(empty + sa, rs.phase ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            const uint8_t* src = s8 + s8i * kStage8Bytes;
            uint8_t* dst = sA + sa * kStageBytes;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rr = cw * 32 + i * 4 + (lane >> 3);
                const int cc = lane & 7;
#pragma unroll
                for (int kh = 0; kh < kHalves; ++kh) {
                    const uint2 raw = *reinterpret_cast<const uint2*>(src + rr * D + kh * 64 + cc * 8);
                    *reinterpret_cast<uint4*>(dst + kh * kHalfBytes + rr * 128 + ((cc ^ (rr & 7)) << 4)) =
                        e4m3x8_to_bf16x8(raw);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(full + sa);
                mbar_arrive(sempty + s8i);
            }
            ++it;
            r8.next(S8);
            rs.next(SA);
            cur.next();
        }
        if (!ok) raise_abort(abort_flag, p.status);
        if (ok && cw == 0 && lane == 0)
            for (int n = it > SA ? it - SA : 0; n < it; ++n) mbar_wait(empty + n % SA, (n / SA) & 1, nullptr);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem_base, ncols);
}

// Query heads for fp8 scoring (see launch_qsplit).  CTA (row, g) splits the
// heads 4g .. 4g + 3 of one query row, one warp per head (all their loads in
// flight at once), four elements per lane.  The power of two puts the
// head's largest |q| in (224, 448] (e4m3's largest finite value is 448), so
// q1 = e4m3(q * 2^e) and q2 = e4m3(q * 2^e - q1) hold the bf16 value exactly
// unless part of it falls below e4m3's smallest step (2^-9).
__global__ void __launch_bounds__(128) qsplit_kernel(const uint16_t* __restrict__ Q, const float* __restrict__ w,
                                                     int H, int npad, uint8_t* __restrict__ q8,
                                                     float* __restrict__ w8) {
    const int row = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dependency_wait();
    grid_launch_dependents();
    for (int h = blockIdx.y * 4 + warp; h < npad; h += 4 * gridDim.y) {
        uint32_t* o1 = reinterpret_cast<uint32_t*>(q8 + (static_cast<size_t>(row) * 2 * npad + h) * 128);
        uint32_t* o2 = reinterpret_cast<uint32_t*>(q8 + (static_cast<size_t>(row) * 2 * npad + npad + h) * 128);
        if (h >= H) {
            o1[lane] = 0u;
            o2[lane] = 0u;
            if (lane == 0) w8[static_cast<size_t>(row) * npad + h] = 0.f;
            continue;
        }
        const uint2 raw = *reinterpret_cast<const uint2*>(Q + (static_cast<size_t>(row) * H + h) * 128 + lane * 4);
        float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
        float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.f) {
            const int E = static_cast<int>((__float_as_uint(mx) >> 23) & 255u) - 127;   // floor(log2 mx)
            e = 8 - E;                                        // mx * 2^e in [256, 512)
            e = e > 126 ? 126 : (e < -126 ? -126 : e);
            if (mx * __uint_as_float(static_cast<uint32_t>(127 + e) << 23) > 448.f) --e;
        }
        const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);     // 2^e, exact
        uint32_t p1 = 0, p2 = 0;
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
            const float2 a = make_float2(v[i] * up, v[i + 1] * up);
            const __nv_fp8x2_storage_t c1 = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
            const float2 f1 = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(c1, __NV_E4M3)));
            const float2 r = make_float2(a.x - f1.x, a.y - f1.y);              // exact
            const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3);
            p1 |= static_cast<uint32_t>(c1) << (8 * i);
            p2 |= static_cast<uint32_t>(c2) << (8 * i);
        }
        o1[lane] = p1;
        o2[lane] = p2;
        if (lane == 0)
            w8[static_cast<size_t>(row) * npad + h] =
                w[static_cast<size_t>(row) * H + h] * __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    }
}

template <int MODE, bool E4M3, int D, int BV = kBlocksPlain>
cudaError_t launch_t(const CUtensorMap& amap, const CUtensorMap& qmap, const ScoreParams& p, int grid,
                     cudaStream_t s) {
    const size_t smem = score_smem_bytes(MODE, E4M3, D, p.npad, p.stages, p.stages8);
    // the swizzled TMA destinations (operand stages, query heads) start on 1024-byte boundaries
    const Layout L = score_layout(MODE, E4M3, D, p.npad, p.stages, p.stages8);
    if ((L.a | L.q) & 1023u) return cudaErrorInvalidValue;
    auto* fn = score_kernel<MODE, E4M3, D, BV>;
    cudaError_t e = smem_limit(reinterpret_cast<const void*>(fn), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(score_threads(MODE, E4M3, D));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // prologue overlaps
    attr[0].val.programmaticStreamSerializationAllowed = 1;            // the previous kernel
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fn, amap, qmap, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_qsplit(const uint16_t* Q, const float* w, int n_q, int H, int npad, uint8_t* q8,
                          float* w8, cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_q), static_cast<unsigned>((npad + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qsplit_kernel, Q, w, H, npad, q8, w8);
}

size_t score_smem_bytes(int mode, bool e4m3, int d, int npad, int stages, int stages8) {
    const size_t need = score_layout(mode, e4m3, d, npad, stages, stages8).total + 1024;
    const size_t lo = ctas_per_sm(mode, e4m3, d, npad) == 2 ? kMinSmem2 : kMinSmem;
    return need < lo ? lo : need;
}

// Operand stages (and e4m3 staging stages) as many as fit the CTA's share of
// shared memory (the e4m3 converter path keeps two bf16 operand stages and
// spends the rest on staging), and the accumulators that fit its TMEM share.
// Returns the CTAs per SM.
int score_config(int mode, bool e4m3, int d, int npad, int* stages, int* stages8, int* nacc) {
    const int per_sm = ctas_per_sm(mode, e4m3, d, npad);
    const uint32_t budget = static_cast<uint32_t>(per_sm == 2 ? kSmem2 : kMaxSmem);
    *stages = 0;
    *stages8 = 0;
    *nacc = acc_count(acc_width(mode, e4m3, d, npad), per_sm);
    if (!e4m3 || uses_f8(mode, e4m3, d)) {
        for (int s = 2; s <= kMaxStages; ++s)
            if (score_layout(mode, e4m3, d, npad, s, 0).total + 1024 <= budget) *stages = s;
        return per_sm;
    }
    for (int s8 = 2; s8 <= kMaxStages; ++s8)
        if (score_layout(mode, true, d, npad, 2, s8).total + 1024 <= budget) {
            *stages = 2;
            *stages8 = s8;
        }
    return per_sm;
}

cudaError_t launch_score(int mode, bool e4m3, int d, const CUtensorMap& amap, const CUtensorMap& qmap,
                         const ScoreParams& p, int grid, cudaStream_t s) {
    if (mode == kScoreBlocks) {
        if (p.app)   // the decode step: whole rows per CTA (fuse = 1)
            return d == 128 ? launch_t<kScoreBlocks, false, 128, kBlocksAppend>(amap, qmap, p, grid, s)
                            : launch_t<kScoreBlocks, false, 64, kBlocksAppend>(amap, qmap, p, grid, s);
        if (p.cp)
            return d == 128 ? launch_t<kScoreBlocks, false, 128, kBlocksShard>(amap, qmap, p, grid, s)
                            : launch_t<kScoreBlocks, false, 64, kBlocksShard>(amap, qmap, p, grid, s);
        if (p.parent && p.parent_n)
            return d == 128 ? launch_t<kScoreBlocks, false, 128, kBlocksGathered>(amap, qmap, p, grid, s)
                            : launch_t<kScoreBlocks, false, 64, kBlocksGathered>(amap, qmap, p, grid, s);
        if (p.parent)
            return d == 128 ? launch_t<kScoreBlocks, false, 128, kBlocksMasked>(amap, qmap, p, grid, s)
                            : launch_t<kScoreBlocks, false, 64, kBlocksMasked>(amap, qmap, p, grid, s);
        return d == 128 ? launch_t<kScoreBlocks, false, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreBlocks, false, 64>(amap, qmap, p, grid, s);
    }
    if (mode == kScoreFlat) {
        if (e4m3)
            return d == 128 ? launch_t<kScoreFlat, true, 128>(amap, qmap, p, grid, s)
                            : launch_t<kScoreFlat, true, 64>(amap, qmap, p, grid, s);
        return d == 128 ? launch_t<kScoreFlat, false, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreFlat, false, 64>(amap, qmap, p, grid, s);
    }
    if (e4m3)
        return d == 128 ? launch_t<kScoreHisa, true, 128>(amap, qmap, p, grid, s)
                        : launch_t<kScoreHisa, true, 64>(amap, qmap, p, grid, s);
    return d == 128 ? launch_t<kScoreHisa, false, 128>(amap, qmap, p, grid, s)
                    : launch_t<kScoreHisa, false, 64>(amap, qmap, p, grid, s);
}

}  // namespace hisa
