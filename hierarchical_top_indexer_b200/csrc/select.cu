// Exact top-k selection with ties broken toward the lower index.
//
// HISA keeps the top-m blocks by representative score and then the top-k
// tokens of the kept blocks (gptget.net summary, "Methodology"; Chinese
// summary, method details); the flat scan keeps the top-k of all visible
// tokens.  All of them use this kernel on 32-bit order-preserving score keys
// (key 0 = empty / masked slot).
//
// One thread-block cluster per row; CTA r of the cluster stages the r-th
// contiguous chunk of the row's slots in its shared memory, and the CTAs
// exchange partial results through distributed shared memory:
//   1. count, min and max of the nonzero keys (reduced on rank 0);
//   2. a 2048-bin histogram over [min, max] (bins of 2^shift keys, reduced
//      on rank 0) locates the bin of the k-th largest key; a crowded bin
//      narrows the range and the histogram repeats;
//   3. the bin's members are gathered on rank 0 and ranked by counting,
//      which gives the exact k-th largest key T and how many keys equal to
//      T belong to the top k;
//   4. each CTA counts its keys above / equal to T; the counts of lower
//      ranks give its output offset and its share of the keys == T (lowest
//      slots first); an ordered compaction (warp-contiguous slot ranges,
//      ballots for in-warp ranks) writes the kept slots in ascending order.
// Slots are laid out in ascending token order, so the output is ascending in
// token index, followed by -1 padding.
#include <cooperative_groups.h>

#include "hisa_kernels.cuh"

namespace cg = cooperative_groups;

namespace hisa {

namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxChunk = 32768;    // slots staged per CTA
constexpr int kMaxCluster = 8;
constexpr int kBins = 2048;
constexpr int kBinBits = 11;
constexpr int kMembersCap = 1024;   // bin members ranked directly

struct SelShared {
    uint32_t hist[kBins];                         // local histogram / copy of the reduced one
    uint32_t hist_red[kBins];                     // rank 0: cluster-wide histogram
    unsigned long long members[kMembersCap];      // rank 0: gathered bin members
    unsigned long long mloc[kMembersCap];         // local copy of the members
    uint32_t stats[kMaxCluster][3];               // rank 0: per-rank count, min, max
    uint32_t counts[kMaxCluster][2];              // rank 0: per-rank keys above / equal to T
    uint32_t member_count;                        // rank 0
    uint32_t warp_a[kSelWarps];
    uint32_t warp_b[kSelWarps];
    uint32_t warp_c[kSelWarps];
    uint32_t warp_d[kSelWarps];
    uint32_t bcast[8];
};

// Where the CTA's keys come from (slots are CTA-local: 0 .. nl-1).
struct Keys {
    const uint32_t* smem;   // staged keys (or null)
    const uint32_t* g;      // keys in global memory
    const float* x;         // raw fp32 values (kSelF32Rows)
    __device__ __forceinline__ uint32_t operator()(int c) const {
        if (smem) return smem[c];
        if (x) return score_key(x[c]);
        return g[c];
    }
};

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exact k-th largest nonzero key T over the cluster's keys and the number of
// keys == T inside the top k (requires more than k nonzero keys).
__device__ void cluster_kth_key(cg::cluster_group& cluster, const Keys& keys, int nl, int slot0, int k,
                                uint32_t lo, uint32_t hi, SelShared& sh, uint32_t& T, int& take_eq) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const unsigned rank = cluster.block_rank();
    uint32_t* red = cluster.map_shared_rank(sh.hist_red, 0);
    int krem = k;
    for (;;) {
        const uint32_t span = hi - lo;
        const int shift = span == 0 ? 0 : max(0, 32 - __clz(span) - kBinBits);
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = 0;
        __syncthreads();
        for (int c = tid; c < nl; c += kSelThreads) {
            const uint32_t x = keys(c);
            if (x != 0u && x >= lo && x <= hi) atomicAdd(&sh.hist[(x - lo) >> shift], 1u);
        }
        __syncthreads();
        for (int i = tid; i < kBins; i += kSelThreads)
            if (sh.hist[i]) atomicAdd(red + i, sh.hist[i]);
        cluster.sync();
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist[i] = red[i];
        __syncthreads();
        // highest bin whose suffix count reaches krem: each thread owns 2 bins
        const int b0 = kBins - 1 - 2 * tid;   // thread 0 owns the top bins
        const uint32_t l0 = sh.hist[b0], l1 = sh.hist[b0 - 1];
        const uint32_t lsum = l0 + l1;
        uint32_t incl = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) sh.warp_a[warp] = incl;
        __syncthreads();
        uint32_t before = 0;
        for (int w = 0; w < warp; ++w) before += sh.warp_a[w];
        const uint32_t excl = before + incl - lsum;
        const uint32_t kr = static_cast<uint32_t>(krem);
        if (excl < kr && kr <= excl + lsum) {
            if (excl + l0 >= kr) {
                sh.bcast[0] = static_cast<uint32_t>(b0);
                sh.bcast[1] = kr - excl;
                sh.bcast[2] = l0;
            } else {
                sh.bcast[0] = static_cast<uint32_t>(b0 - 1);
                sh.bcast[1] = kr - excl - l0;
                sh.bcast[2] = l1;
            }
        }
        __syncthreads();
        const uint32_t bin = sh.bcast[0];
        krem = static_cast<int>(sh.bcast[1]);
        const uint32_t nmem = sh.bcast[2];
        const uint32_t blo = lo + (bin << shift);
        const uint32_t bhi = shift == 0 ? blo : blo + ((1u << shift) - 1u);
        __syncthreads();
        if (shift == 0) {          // a single key value: it is T
            T = blo;
            take_eq = krem;
            return;
        }
        if (nmem <= static_cast<uint32_t>(kMembersCap)) {
            unsigned long long* rmem = cluster.map_shared_rank(sh.members, 0);
            uint32_t* rcnt = cluster.map_shared_rank(&sh.member_count, 0);
            for (int c = tid; c < nl; c += kSelThreads) {
                const uint32_t x = keys(c);
                if (x >= blo && x <= bhi && x != 0u) {
                    const uint32_t at = atomicAdd(rcnt, 1u);
                    rmem[at] = (static_cast<unsigned long long>(x) << 32) | static_cast<uint32_t>(slot0 + c);
                }
            }
            cluster.sync();
            const int cnt = static_cast<int>(*rcnt);
            for (int i = tid; i < cnt; i += kSelThreads) sh.mloc[i] = rmem[i];
            __syncthreads();
            for (int i = tid; i < cnt; i += kSelThreads) {
                const uint32_t xi = static_cast<uint32_t>(sh.mloc[i] >> 32);
                int above = 0, equal = 0;
                for (int j = 0; j < cnt; ++j) {
                    const uint32_t xj = static_cast<uint32_t>(sh.mloc[j] >> 32);
                    above += xj > xi;
                    equal += xj == xi;
                }
                // xi is T iff the krem-th position falls in xi's run of equal keys
                if (above < krem && krem <= above + equal) {
                    sh.bcast[4] = xi;
                    sh.bcast[5] = static_cast<uint32_t>(krem - above);
                }
            }
            __syncthreads();
            T = sh.bcast[4];
            take_eq = static_cast<int>(sh.bcast[5]);
            __syncthreads();
            return;
        }
        // too many keys in the bin: narrow the range and repeat
        cluster.sync();                 // everyone has read the reduced histogram
        if (rank == 0)
            for (int i = tid; i < kBins; i += kSelThreads) sh.hist_red[i] = 0;
        cluster.sync();
        lo = blo;
        hi = bhi;
    }
}

// Block-wide exclusive scan helper for the per-warp totals in warp_a / warp_b.
// Ordered compaction of the CTA's keys: keeps keys > T plus keys == T whose
// cluster-wide rank among equal keys is below take_eq.  eq_base = keys == T
// in lower ranks, out_base = kept keys in lower ranks.  Calls emit(pos, slot,
// key).  Returns the number kept by this CTA.
template <class Emit>
__device__ int compact(const Keys& keys, int nl, uint32_t T, int take_eq, uint32_t eq_base,
                       uint32_t out_base, SelShared& sh, Emit emit) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_warp = ((nl + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int w0 = warp * per_warp;
    const int w1 = min(nl, w0 + per_warp);
    uint32_t gt = 0, eq = 0;
    for (int base = w0; base < w1; base += 32) {
        const int c = base + lane;
        const uint32_t x = c < w1 ? keys(c) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, x != 0u && x > T));
        eq += __popc(__ballot_sync(0xffffffffu, x != 0u && x == T));
    }
    if (lane == 0) {
        sh.warp_a[warp] = gt;
        sh.warp_b[warp] = eq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t eq_before = eq_base, off = out_base;
        for (int w = 0; w < kSelWarps; ++w) {
            const uint32_t e = sh.warp_b[w];
            const int room = take_eq - static_cast<int>(eq_before);
            const uint32_t take = room <= 0 ? 0u : (static_cast<uint32_t>(room) < e ? room : e);
            sh.warp_c[w] = eq_before;
            sh.warp_d[w] = off;
            eq_before += e;
            off += sh.warp_a[w] + take;
        }
        sh.bcast[6] = off - out_base;
    }
    __syncthreads();
    uint32_t eq_run = sh.warp_c[warp];
    uint32_t pos = sh.warp_d[warp];
    const unsigned lt = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
        const int c = base + lane;
        const uint32_t x = c < w1 ? keys(c) : 0u;
        const bool is_gt = x != 0u && x > T;
        const bool is_eq = x != 0u && x == T;
        const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t eq_rank = eq_run + __popc(eqb & lt);
        const bool sel = is_gt || (is_eq && eq_rank < static_cast<uint32_t>(take_eq));
        const unsigned selb = __ballot_sync(0xffffffffu, sel);
        if (sel) emit(static_cast<int>(pos + __popc(selb & lt)), c, x);
        eq_run += __popc(eqb);
        pos += __popc(selb);
    }
    const int total = static_cast<int>(sh.bcast[6]);
    __syncthreads();
    return total;
}

// Keys of the CTA's chunk with T known: counts above / equal to T.
__device__ void count_vs(const Keys& keys, int nl, uint32_t T, SelShared& sh, uint32_t& gt_out,
                         uint32_t& eq_out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t gt = 0, eq = 0;
    for (int c = threadIdx.x; c < nl; c += kSelThreads) {
        const uint32_t x = keys(c);
        gt += x != 0u && x > T;
        eq += x != 0u && x == T;
    }
    gt = warp_sum(gt);
    eq = warp_sum(eq);
    if (lane == 0) {
        sh.warp_c[warp] = gt;
        sh.warp_d[warp] = eq;
    }
    __syncthreads();
    gt_out = eq_out = 0;
    for (int w = 0; w < kSelWarps; ++w) {
        gt_out += sh.warp_c[w];
        eq_out += sh.warp_d[w];
    }
    __syncthreads();
}

template <bool STAGE>
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelectParams p) {
    extern __shared__ uint32_t staged[];
    __shared__ SelShared sh;
    grid_dependency_wait();
    grid_launch_dependents();
    cg::cluster_group cluster = cg::this_cluster();
    const int csize = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.x / csize;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    // ---- row geometry (identical on every rank of the cluster)
    int n = 0, kk = p.k, b = 0, t = 0, nb = 0;
    bool bad = false;
    if (p.mode == kSelF32Rows) {
        n = p.n;
    } else if (p.mode == kSelHisaTokens) {
        const int4 pl = p.plan[row];
        b = pl.x;
        t = pl.y;
        bad = t < 0;
        n = pl.z * p.B;
    } else {
        t = query_position(p.q_seq, p.q_pos, p.len, p.batch, p.cap, row, &b);
        bad = t < 0;
        if (p.mode == kSelBlocks) {
            nb = t / p.B + 1;
            n = nb - 1;          // every block but the own one competes
            kk = p.m - 1;        // for m - 1 places
        } else {
            n = t + 1;
        }
    }

    if (bad || (p.mode == kSelBlocks && nb <= p.m && !p.tree)) {
        if (rank == 0) {
            if (p.mode == kSelBlocks) {
                // bad row: nothing kept; short row: every visible block kept
                const int keep = bad ? 0 : nb;
                for (int r = tid; r < p.mm; r += kSelThreads) {
                    const int v = r < keep ? r : -1;
                    p.blocks[static_cast<size_t>(row) * p.mm + r] = v;
                    if (p.blocks_out) p.blocks_out[static_cast<size_t>(row) * p.mm + r] = v;
                }
                if (tid == 0) {
                    p.nblocks[row] = keep;
                    if (p.nblocks_out) p.nblocks_out[row] = keep;
                    p.plan[row] = make_int4(b, bad ? -1 : t, keep, 0);
                    if (bad) set_status(p.status, HISA_DEV_BAD_QUERY);
                }
            } else {
                for (int r = tid; r < p.k; r += kSelThreads) {
                    p.idx[static_cast<size_t>(row) * p.k + r] = -1;
                    if (p.scores) p.scores[static_cast<size_t>(row) * p.k + r] = __int_as_float(0x7fc00000);
                }
                if (tid == 0 && p.mode != kSelHisaTokens) set_status(p.status, HISA_DEV_BAD_QUERY);
            }
        }
        cluster.sync();
        return;
    }

    // ---- this rank's chunk of slots
    const int chunk = ((n + csize - 1) / csize + 127) & ~127;
    const int s0 = min(n, rank * chunk);
    const int nl = min(n, s0 + chunk) - s0;
    Keys keys{nullptr, nullptr, nullptr};
    if (p.mode == kSelF32Rows) keys.x = p.x + static_cast<size_t>(row) * p.n + s0;
    else keys.g = p.keys + static_cast<size_t>(row) * p.ldk + s0;

    if (rank == 0) {
        for (int i = tid; i < kBins; i += kSelThreads) sh.hist_red[i] = 0;
        if (tid == 0) sh.member_count = 0;
    }

    // ---- pass 1: stage, count, min, max
    uint32_t cnt = 0, mn = 0xFFFFFFFFu, mx = 0u;
    if (keys.g) {
        const uint4* g4 = reinterpret_cast<const uint4*>(keys.g);   // s0, ldk: multiples of 128
        const int n4 = (nl + 3) >> 2;
#pragma unroll 4
        for (int c4 = tid; c4 < n4; c4 += kSelThreads) {
            const uint4 v = __ldcg(g4 + c4);
            const uint32_t xs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 4 * c4 + j;
                const uint32_t x = c < nl ? xs[j] : 0u;
                if (STAGE && c < nl) staged[c] = x;
                if (x != 0u) {
                    ++cnt;
                    mn = min(mn, x);
                    mx = max(mx, x);
                }
            }
        }
    } else {
        for (int c = tid; c < nl; c += kSelThreads) {
            const uint32_t x = keys(c);
            if (STAGE) staged[c] = x;
            if (x != 0u) {
                ++cnt;
                mn = min(mn, x);
                mx = max(mx, x);
            }
        }
    }
    cnt = warp_sum(cnt);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        sh.warp_a[warp] = cnt;
        sh.warp_b[warp] = mn;
        sh.warp_c[warp] = mx;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t c0 = 0, m0 = 0xFFFFFFFFu, m1 = 0u;
        for (int w = 0; w < kSelWarps; ++w) {
            c0 += sh.warp_a[w];
            m0 = min(m0, sh.warp_b[w]);
            m1 = max(m1, sh.warp_c[w]);
        }
        uint32_t* rs = cluster.map_shared_rank(&sh.stats[rank][0], 0);
        rs[0] = c0;
        rs[1] = m0;
        rs[2] = m1;
    }
    if (STAGE) keys.smem = staged;
    cluster.sync();
    uint32_t nvalid = 0;
    mn = 0xFFFFFFFFu;
    mx = 0u;
    {
        const uint32_t* rs = cluster.map_shared_rank(&sh.stats[0][0], 0);
        for (int r = 0; r < csize; ++r) {
            nvalid += rs[3 * r];
            mn = min(mn, rs[3 * r + 1]);
            mx = max(mx, rs[3 * r + 2]);
        }
    }

    // ---- threshold
    uint32_t T = 0;
    int take_eq = 0;
    if (kk > 0 && nvalid > static_cast<uint32_t>(kk))
        cluster_kth_key(cluster, keys, nl, s0, kk, mn, mx, sh, T, take_eq);

    // ---- offsets from the lower ranks
    uint32_t eq_base = 0, out_base = 0, kept_total = 0;
    if (kk > 0) {
        uint32_t gt_l, eq_l;
        count_vs(keys, nl, T, sh, gt_l, eq_l);
        if (tid == 0) {
            uint32_t* rc = cluster.map_shared_rank(&sh.counts[rank][0], 0);
            rc[0] = gt_l;
            rc[1] = eq_l;
        }
        cluster.sync();
        const uint32_t* rc = cluster.map_shared_rank(&sh.counts[0][0], 0);
        uint32_t eqb = 0, outb = 0;
        for (int r = 0; r < csize; ++r) {
            const uint32_t g = rc[2 * r], e = rc[2 * r + 1];
            const int room = take_eq - static_cast<int>(eqb);
            const uint32_t take = room <= 0 ? 0u : (static_cast<uint32_t>(room) < e ? room : e);
            if (r == rank) {
                eq_base = eqb;
                out_base = outb;
            }
            eqb += e;
            outb += g + take;
        }
        kept_total = outb;
    }

    // ---- outputs
    if (p.mode == kSelBlocks) {
        int32_t* out = p.blocks + static_cast<size_t>(row) * p.mm;
        int32_t* dbg = p.blocks_out ? p.blocks_out + static_cast<size_t>(row) * p.mm : nullptr;
        if (kk > 0)
            compact(keys, nl, T, take_eq, eq_base, out_base, sh, [&](int pos, int c, uint32_t) {
                out[pos] = s0 + c;
                if (dbg) dbg[pos] = s0 + c;
            });
        if (rank == 0) {
            for (int r = static_cast<int>(kept_total) + tid; r < p.mm; r += kSelThreads) {
                const int v = r == static_cast<int>(kept_total) ? nb - 1 : -1;   // own block last
                out[r] = v;
                if (dbg) dbg[r] = v;
            }
            if (tid == 0) {
                const int keep = static_cast<int>(kept_total) + 1;
                p.nblocks[row] = keep;
                if (p.nblocks_out) p.nblocks_out[row] = keep;
                p.plan[row] = make_int4(b, t, keep, 0);
            }
        }
    } else {
        int32_t* idx = p.idx + static_cast<size_t>(row) * p.k;
        float* sc = p.scores ? p.scores + static_cast<size_t>(row) * p.k : nullptr;
        const int32_t* blk =
            p.mode == kSelHisaTokens ? p.blocks + static_cast<size_t>(row) * p.mm : nullptr;
        const int Bsz = p.B;
        compact(keys, nl, T, take_eq, eq_base, out_base, sh, [&](int pos, int c, uint32_t x) {
            const int slot = s0 + c;
            idx[pos] = (blk ? blk[slot / Bsz] * Bsz + slot % Bsz : slot) + p.id_off;
            if (sc) sc[pos] = key_score(x);
        });
        if (rank == 0)
            for (int r = static_cast<int>(kept_total) + tid; r < p.k; r += kSelThreads) {
                idx[r] = -1;
                if (sc) sc[r] = __int_as_float(0x7fc00000);
            }
    }
    cluster.sync();   // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------ single-CTA rows
//
// Rows of up to kRowKeys slots: one CTA of NT threads; thread t holds the KPT
// consecutive slots t*KPT .. t*KPT + KPT - 1 of the row in registers, so every
// pass over the row (count / min / max, histogram, bin members, compaction)
// reads registers, and the ordered compaction needs a single block-wide scan
// of a thread's (greater-than, equal-to) counts.  Every block-wide scan or
// reduction is one barrier: warp totals go to shared memory and each warp
// then reduces or scans all of them with shuffles.
// NT = 1024 serves few rows (up to two per SM: more warps per row shorten
// each phase), NT = 512 many rows (more CTAs per SM).

constexpr int kRowBlocks = 2048;   // kept-block ids staged in shared memory

template <int NT>
struct RowShared {
    static constexpr int kWarps = NT / 32;
    int32_t blk[kRowBlocks];
    uint32_t hist[kBins];
    unsigned long long members[kMembersCap];
    uint32_t wa[kWarps];
    uint32_t wb[kWarps];
    uint32_t wc[kWarps];
    uint32_t wd[kWarps];     // the compaction's scan (wa..wc may still be read then)
    uint32_t nmem;
    uint32_t bc[8];
};

// Exclusive block scan of one value per thread (NT threads, thread order);
// *total = the sum over the block.  One barrier; wtot must not be read or
// written by another scan until the caller's next barrier.
template <int NT>
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* wtot, uint32_t* total) {
    constexpr int NW = NT / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    // every warp scans the NW warp totals
    uint32_t t = lane < NW ? wtot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += x;
    }
    *total = __shfl_sync(0xffffffffu, ti, 31);
    const uint32_t before = __shfl_sync(0xffffffffu, ti - t, warp);   // exclusive prefix of this warp
    return before + incl - v;
}

// Outputs of a row are staged in shared memory and written out in order with
// 16-byte stores when the row's k entries fit (stage_k = k, a multiple of 4;
// 0 = write each entry where it goes).
// MODE >= 0 fixes the selection mode at compile time (the token rows of the
// HISA path, so that their code carries no other mode's branches); -1 reads
// it from p.
template <int NT, int KPT, int MODE>
__global__ void __launch_bounds__(NT, NT >= 1024 ? 1 : (NT >= 512 ? 2 : 4)) select_row_kernel(const SelectParams p, int stage_k) {
    static_assert(KPT % 4 == 0, "slots per thread in 16-byte groups");
    static_assert(NT * KPT <= 65535, "packed (gt, eq) counts fit 16 bits each");
    constexpr int kBinsPer = kBins / NT;   // histogram bins each thread scans
    static_assert(kBins % NT == 0, "bins split evenly over the threads");
    __shared__ RowShared<NT> sh;
    extern __shared__ __align__(16) int32_t stage_out[];   // [stage_k] ids, then [stage_k] scores
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int mode = MODE >= 0 ? MODE : p.mode;
    // token rows: this thread's keys load before the row's plan is read (its
    // slot count masks them later), so that the two L2 round trips overlap;
    // the loads stay within the row's ldk slots
    uint4 kpre[KPT / 4];
    if (MODE == kSelHisaTokens) {
        const uint4* g4 = reinterpret_cast<const uint4*>(p.keys + static_cast<size_t>(row) * p.ldk + tid * KPT);
#pragma unroll
        for (int q = 0; q < KPT / 4; ++q)
            kpre[q] = tid * KPT + 4 * q < p.ldk ? __ldg(g4 + q) : make_uint4(0u, 0u, 0u, 0u);
    }

    int n = 0, kk = p.k, b = 0, t = 0, nb = 0, cp_own = 0;
    bool bad = false;
    if (mode == kSelF32Rows) {
        n = p.n;
    } else if (mode == kSelMerge) {
        n = p.lists * p.n;
    } else if (mode == kSelHisaTokens) {
        const int4 pl = p.plan[row];
        b = pl.x;
        t = pl.y;
        bad = t < 0;
        n = pl.z * p.B;
    } else if (mode == kSelCpBlocks) {
        // the shard's visible blocks but the own one compete for m - 1 places
        nb = cp_visible_blocks(p.q_seq, p.q_pos, p.len, p.batch, p.cap, p.B, p.id_off * p.B, row, &b,
                               &cp_own, &t);
        bad = nb < 0;
        n = bad ? 0 : nb - cp_own;
        kk = p.m - 1;
    } else {
        t = query_position(p.q_seq, p.q_pos, p.len, p.batch, p.cap, row, &b);
        bad = t < 0;
        if (mode == kSelBlocks) {
            nb = t / p.B + 1;
            n = nb - 1;
            kk = p.m - 1;
        } else {
            n = t + 1;
        }
    }
    if (bad || (mode == kSelBlocks && nb <= p.m && !p.tree)) {
        if (mode == kSelBlocks) {
            const int keep = bad ? 0 : nb;
            for (int r = tid; r < p.mm; r += NT) {
                const int v = r < keep ? r : -1;
                p.blocks[static_cast<size_t>(row) * p.mm + r] = v;
                if (p.blocks_out) p.blocks_out[static_cast<size_t>(row) * p.mm + r] = v;
            }
            if (tid == 0) {
                p.nblocks[row] = keep;
                if (p.nblocks_out) p.nblocks_out[row] = keep;
                p.plan[row] = make_int4(b, bad ? -1 : t, keep, 0);
                if (bad) set_status(p.status, HISA_DEV_BAD_QUERY);
            }
        } else {
            for (int r = tid; r < p.k; r += NT) {
                p.idx[static_cast<size_t>(row) * p.k + r] = -1;
                if (p.scores) p.scores[static_cast<size_t>(row) * p.k + r] = __int_as_float(0x7fc00000);
            }
            if (tid == 0 && bad && mode != kSelHisaTokens) set_status(p.status, HISA_DEV_BAD_QUERY);
        }
        return;
    }

    // kept-block ids of a HISA row (slot c belongs to block blk[c / B])
    const bool blk_smem = mode == kSelHisaTokens && p.mm <= kRowBlocks;
    if (blk_smem)
        for (int r = tid; r < p.mm; r += NT) sh.blk[r] = p.blocks[static_cast<size_t>(row) * p.mm + r];
    for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0u;
    if (tid == 0) sh.nmem = 0u;

    // 1. this thread's slots c0 .. c0 + KPT - 1 (key 0 past n); count, min, max
    const int c0 = tid * KPT;
    // slot c of a merged row: list c / n, entry c % n
    auto merge_at = [&](int c) {
        const int l = c / p.n;
        return (static_cast<size_t>(l) * p.rows + row) * p.n + (c - l * p.n);
    };
    uint32_t x[KPT];
    if (mode == kSelF32Rows || mode == kSelMerge) {
        const float* xr = p.x + static_cast<size_t>(row) * p.n;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
            const int c = c0 + e;
            uint32_t v = 0u;
            if (c < n) {
                if (mode == kSelMerge) {
                    const size_t o = merge_at(c);
                    v = p.ids[o] < 0 ? 0u : score_key(p.x[o]);   // an empty entry never competes
                } else {
                    v = score_key(xr[c]);
                }
            }
            x[e] = v;
        }
    } else {
        // rows are ldk (a multiple of 128) keys apart: a 4-key group that
        // starts below n lies inside the row
        const uint4* g4 = reinterpret_cast<const uint4*>(p.keys + static_cast<size_t>(row) * p.ldk + c0);
#pragma unroll
        for (int q = 0; q < KPT / 4; ++q) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (MODE == kSelHisaTokens) v = kpre[q];
            else if (c0 + 4 * q < n) v = __ldg(g4 + q);   // L1 keeps the half of each sector the next load uses
            x[4 * q] = c0 + 4 * q < n ? v.x : 0u;
            x[4 * q + 1] = c0 + 4 * q + 1 < n ? v.y : 0u;
            x[4 * q + 2] = c0 + 4 * q + 2 < n ? v.z : 0u;
            x[4 * q + 3] = c0 + 4 * q + 3 < n ? v.w : 0u;
        }
    }
    uint32_t cnt = 0, mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
        const uint32_t v = x[e];
        cnt += v != 0u;
        mn = v != 0u ? min(mn, v) : mn;
        mx = max(mx, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        sh.wa[warp] = cnt;
        sh.wb[warp] = mn;
        sh.wc[warp] = mx;
    }
    __syncthreads();
    {
        constexpr int NW = NT / 32;
        cnt = lane < NW ? sh.wa[lane] : 0u;
        mn = lane < NW ? sh.wb[lane] : 0xFFFFFFFFu;
        mx = lane < NW ? sh.wc[lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
    }
    const uint32_t nvalid = cnt;

    // 2-3. the k-th largest key T and how many keys == T are kept: a
    // 2048-bin histogram over [lo, hi] finds the bin of the k-th key; a bin of
    // at most kMembersCap keys is ranked by counting, a crowded one becomes
    // the next [lo, hi]
    uint32_t T = 0;
    int take_eq = 0;
    if (kk > 0 && nvalid > static_cast<uint32_t>(kk)) {
        uint32_t lo = mn, hi = mx;
        int krem = kk;
        for (;;) {
            const uint32_t span = hi - lo;
            const int shift = span == 0 ? 0 : max(0, 32 - __clz(span) - kBinBits);
#pragma unroll
            for (int e = 0; e < KPT; ++e) {
                const uint32_t v = x[e];
                if (v != 0u && v >= lo && v <= hi) atomicAdd(&sh.hist[(v - lo) >> shift], 1u);
            }
            __syncthreads();
            // thread t owns kBinsPer consecutive bins from the top (highest first)
            const int b0 = kBins - 1 - kBinsPer * tid;
            uint32_t hs[kBinsPer], loc = 0;
#pragma unroll
            for (int q = 0; q < kBinsPer; ++q) {
                hs[q] = sh.hist[b0 - q];
                loc += hs[q];
            }
            uint32_t tot;
            const uint32_t excl = block_scan<NT>(loc, sh.wc, &tot);
            const uint32_t kr = static_cast<uint32_t>(krem);
            if (excl < kr && kr <= excl + loc) {
                uint32_t run = excl;
#pragma unroll
                for (int q = 0; q < kBinsPer; ++q) {
                    if (run < kr && kr <= run + hs[q]) {
                        sh.bc[0] = static_cast<uint32_t>(b0 - q);
                        sh.bc[1] = kr - run;
                        sh.bc[2] = hs[q];
                    }
                    run += hs[q];
                }
            }
            __syncthreads();
            const uint32_t bin = sh.bc[0];
            krem = static_cast<int>(sh.bc[1]);
            const uint32_t nmem = sh.bc[2];
            const uint32_t blo = lo + (bin << shift);
            const uint32_t bhi = shift == 0 ? blo : blo + ((1u << shift) - 1u);
            if (shift == 0) {
                T = blo;
                take_eq = krem;
                break;
            }
            if (nmem <= static_cast<uint32_t>(kMembersCap)) {
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const uint32_t v = x[e];
                    if (v != 0u && v >= blo && v <= bhi) {
                        const uint32_t at = atomicAdd(&sh.nmem, 1u);
                        sh.members[at] = (static_cast<unsigned long long>(v) << 32) | static_cast<uint32_t>(c0 + e);
                    }
                }
                __syncthreads();
                const int m = static_cast<int>(sh.nmem);
                for (int i = tid; i < m; i += NT) {
                    const uint32_t xi = static_cast<uint32_t>(sh.members[i] >> 32);
                    int above = 0, equal = 0;
                    for (int j = 0; j < m; ++j) {
                        const uint32_t xj = static_cast<uint32_t>(sh.members[j] >> 32);
                        above += xj > xi;
                        equal += xj == xi;
                    }
                    if (above < krem && krem <= above + equal) {
                        sh.bc[4] = xi;
                        sh.bc[5] = static_cast<uint32_t>(krem - above);
                    }
                }
                __syncthreads();
                T = sh.bc[4];
                take_eq = static_cast<int>(sh.bc[5]);
                break;
            }
            // crowded bin: narrow the range and repeat (nobody reads the
            // histogram after the barrier above)
            lo = blo;
            hi = bhi;
            for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0u;
            __syncthreads();
        }
    }

    // 4. ordered compaction: one scan of the packed (> T, == T) counts gives
    // each thread its first output position and its first equal-key rank
    const bool any = kk > 0;
    uint32_t gt = 0, eq = 0;
    if (any) {
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
            gt += x[e] != 0u && x[e] > T;
            eq += x[e] != 0u && x[e] == T;
        }
    }
    uint32_t tot;
    const uint32_t excl = block_scan<NT>((gt << 16) | eq, sh.wd, &tot);
    const uint32_t gt_before = excl >> 16, eq_before = excl & 0xFFFFu;
    const uint32_t te = static_cast<uint32_t>(take_eq);
    const int kept = static_cast<int>((tot >> 16) + min(tot & 0xFFFFu, te));

    int32_t* blist = mode == kSelBlocks ? p.blocks + static_cast<size_t>(row) * p.mm : nullptr;
    int32_t* bdbg = mode == kSelBlocks && p.blocks_out ? p.blocks_out + static_cast<size_t>(row) * p.mm : nullptr;
    int32_t* const idx_g = mode != kSelBlocks ? p.idx + static_cast<size_t>(row) * p.k : nullptr;
    float* const sc_g = mode != kSelBlocks && p.scores ? p.scores + static_cast<size_t>(row) * p.k : nullptr;
    // token rows with staging: emit into shared memory, write out below
    const bool staged = stage_k > 0 && mode != kSelBlocks && mode != kSelCpBlocks;
    int32_t* idx = staged ? stage_out : idx_g;
    float* sc = !sc_g ? nullptr : staged ? reinterpret_cast<float*>(stage_out + stage_k) : sc_g;
    const int32_t* blk = mode != kSelHisaTokens ? nullptr
                         : blk_smem ? sh.blk
                                    : p.blocks + static_cast<size_t>(row) * p.mm;
    const int Bsz = p.B;
    const bool pow2 = (Bsz & (Bsz - 1)) == 0;
    const int lgB = __ffs(Bsz) - 1;
    if (any) {
        uint32_t pos = gt_before + min(eq_before, te);
        uint32_t eqr = eq_before;
        // a thread's KPT slots start at a multiple of KPT, so they lie in one
        // kept block when KPT divides B: their ids are consecutive from one lookup
        const bool one_blk = blk && Bsz % KPT == 0;
        const int bi0 = one_blk ? (pow2 ? c0 >> lgB : c0 / Bsz) : 0;
        const int id0 = one_blk ? blk[bi0] * Bsz + (c0 - bi0 * Bsz) + p.id_off : 0;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
            const uint32_t v = x[e];
            const bool is_eq = v != 0u && v == T;
            const bool sel = (v != 0u && v > T) || (is_eq && eqr < te);
            eqr += is_eq;
            const int c = c0 + e;
            const int at = static_cast<int>(pos);
            pos += sel;
            if (!sel) continue;
            if (blist) {
                blist[at] = c;
                if (bdbg) bdbg[at] = c;
            } else {
                if (one_blk) {
                    idx[at] = id0 + e;
                } else if (blk) {
                    const int bi = pow2 ? c >> lgB : c / Bsz;
                    idx[at] = blk[bi] * Bsz + (c - bi * Bsz) + p.id_off;
                } else if (mode == kSelMerge) {
                    idx[at] = p.ids[merge_at(c)];
                } else {
                    idx[at] = c + p.id_off;
                }
                if (sc) sc[at] = key_score(v);
            }
        }
    }
    if (mode == kSelBlocks) {
        for (int r = kept + tid; r < p.mm; r += NT) {
            const int v = r == kept ? nb - 1 : -1;   // own block last
            blist[r] = v;
            if (bdbg) bdbg[r] = v;
        }
        if (tid == 0) {
            const int keep = kept + 1;
            p.nblocks[row] = keep;
            if (p.nblocks_out) p.nblocks_out[row] = keep;
            p.plan[row] = make_int4(b, t, keep, 0);
        }
    } else {
        int r0 = kept;
        if (cp_own) {
            // the shard holds the row's own block: it follows the m - 1 others,
            // marked with an infinite score so that every merge keeps it
            if (tid == 0) {
                idx[r0] = p.id_off + nb - 1;
                if (sc) sc[r0] = __int_as_float(0x7f800000);
            }
            ++r0;
        }
        for (int r = r0 + tid; r < p.k; r += NT) {
            idx[r] = -1;
            if (sc) sc[r] = __int_as_float(0x7fc00000);
        }
        if (staged) {
            __syncthreads();
            const int4* si = reinterpret_cast<const int4*>(stage_out);
            int4* gi = reinterpret_cast<int4*>(idx_g);
            for (int r = tid; r < p.k / 4; r += NT) gi[r] = si[r];
            if (sc_g) {
                const int4* ss = reinterpret_cast<const int4*>(stage_out + stage_k);
                int4* gs = reinterpret_cast<int4*>(sc_g);
                for (int r = tid; r < p.k / 4; r += NT) gs[r] = ss[r];
            }
        }
    }
}

// Token rows whose k outputs (ids and scores) fit in this much shared
// memory, with k a multiple of 4 and 16-byte aligned rows, are staged.
constexpr int kStageBytes = 64 * 1024;

template <int NT, int KPT, int MODE>
cudaError_t launch_row_m(const SelectParams& p, cudaStream_t s) {
    const bool tokens = p.mode != kSelBlocks && p.mode != kSelCpBlocks;
    const int per = p.scores ? 8 : 4;
    const bool aligned16 = (reinterpret_cast<uintptr_t>(p.idx) % 16 == 0) &&
                           (!p.scores || reinterpret_cast<uintptr_t>(p.scores) % 16 == 0);
    const int stage_k = tokens && p.k % 4 == 0 && aligned16 && p.k * per <= kStageBytes ? p.k : 0;
    const size_t smem = static_cast<size_t>(stage_k) * per;
    cudaError_t e = smem_limit(reinterpret_cast<const void*>(select_row_kernel<NT, KPT, MODE>), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.rows));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, select_row_kernel<NT, KPT, MODE>, p, stage_k);
}

template <int NT, int KPT>
cudaError_t launch_row_t(const SelectParams& p, cudaStream_t s) {
    return p.mode == kSelHisaTokens ? launch_row_m<NT, KPT, kSelHisaTokens>(p, s) : launch_row_m<NT, KPT, -1>(p, s);
}

// Threads per row: 256 for rows of at most 1024 slots; otherwise 1024 while
// there are at most two rows per SM, else 512 (rows over 512 * 32 slots keep
// 1024); slots per thread: the fewest that cover the longest row.
cudaError_t launch_row(const SelectParams& p, int max_n, int sms, cudaStream_t s) {
    // short rows (block selection at long contexts, merges): 256 threads, whose
    // barriers and scans are cheaper in a chain of latency-bound phases
    if (max_n <= 256 * 4) return launch_row_t<256, 4>(p, s);
    const bool wide = p.rows <= 2 * sms || max_n > 512 * 32;
    if (wide) {
        if (max_n <= 1024 * 4) return launch_row_t<1024, 4>(p, s);
        if (max_n <= 1024 * 8) return launch_row_t<1024, 8>(p, s);
        if (max_n <= 1024 * 16) return launch_row_t<1024, 16>(p, s);
        return launch_row_t<1024, 24>(p, s);
    }
    if (max_n <= 512 * 8) return launch_row_t<512, 8>(p, s);
    if (max_n <= 512 * 16) return launch_row_t<512, 16>(p, s);
    return launch_row_t<512, 32>(p, s);
}

template <bool STAGE>
cudaError_t launch_t(const SelectParams& p, int csize, int chunk, cudaStream_t s) {
    const size_t smem = STAGE ? static_cast<size_t>(chunk) * sizeof(uint32_t) : 0;
    auto* fn = select_kernel<STAGE>;
    cudaError_t e = smem_limit(reinterpret_cast<const void*>(fn), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.rows * csize));
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, fn, p);
}

// One warp per row: the shard's visible blocks among the row's merged global
// block list, in order (an ordered compaction by ballots).
__global__ void __launch_bounds__(128) cp_localize_kernel(const CpLocalizeParams p) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= p.rows) return;
    int b, own, tl;
    const int vis = cp_visible_blocks(p.q_seq, p.q_pos, p.len, p.batch, p.cap, p.B, p.tok_off, row, &b,
                                      &own, &tl);
    const int blk0 = p.tok_off / p.B;
    const int32_t* kept = p.kept + static_cast<size_t>(row) * p.m;
    int32_t* out = p.blocks + static_cast<size_t>(row) * p.mm;
    const int t = p.q_pos[row];
    const int g_own = t >= 0 ? t / p.B : -2;
    bool has_own = false;
    for (int base = 0; base < p.m; base += 32) {
        const int j = base + lane;
        has_own |= __any_sync(0xffffffffu, j < p.m && kept[j] == g_own);
    }
    const bool valid = vis >= 0 && has_own;
    int cnt = 0;
    if (valid && vis > 0)
        for (int base = 0; base < p.m; base += 32) {
            const int j = base + lane;
            const int g = j < p.m ? kept[j] : -1;
            const bool mine = g >= blk0 && g - blk0 < vis;
            const unsigned bal = __ballot_sync(0xffffffffu, mine);
            const int at = cnt + __popc(bal & ((1u << lane) - 1u));
            if (mine && at < p.mm) out[at] = g - blk0;
            cnt += __popc(bal);
        }
    cnt = min(cnt, p.mm);
    for (int j = cnt + lane; j < p.mm; j += 32) out[j] = -1;
    if (lane == 0) {
        p.nblocks[row] = cnt;
        // the own block is the last kept one on the shard that holds the query
        // position; elsewhere every kept block is visible as a whole
        p.plan[row] = make_int4(b, !valid ? -1 : (own ? tl : p.cap - 1), cnt, 0);
        if (!valid) set_status(p.status, HISA_DEV_BAD_QUERY);
    }
}

}  // namespace

cudaError_t launch_cp_localize(const CpLocalizeParams& p, cudaStream_t s) {
    if (p.rows <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((p.rows + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, cp_localize_kernel, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_select(const SelectParams& p, int max_n, int sms, cudaStream_t s) {
    if (p.rows <= 0) return cudaSuccess;
    if ((p.mode == kSelCpBlocks || p.mode == kSelMerge) && max_n > kRowKeys) return cudaErrorInvalidValue;
    if (max_n <= kRowKeys) {
        const cudaError_t e = launch_row(p, max_n, sms, s);
        return e == cudaSuccess ? cudaGetLastError() : e;
    }
    // cluster size: enough CTAs to stage the longest row, and more while
    // there are SMs to spare; chunks stay at least 1024 slots
    int csize = 1;
    while (csize < kMaxCluster && static_cast<long long>(csize) * kMaxChunk < max_n) csize *= 2;
    while (csize < kMaxCluster && static_cast<long long>(p.rows) * csize * 2 <= sms &&
           max_n / (csize * 2) >= 1024)
        csize *= 2;
    const int chunk = ((max_n + csize - 1) / csize + 127) & ~127;
    cudaError_t e;
    if (chunk <= kMaxChunk) e = launch_t<true>(p, csize, chunk > 0 ? chunk : 128, s);
    else e = launch_t<false>(p, csize, 0, s);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e;
}

}  // namespace hisa
