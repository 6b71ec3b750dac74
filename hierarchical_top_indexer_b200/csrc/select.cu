// Exact top-k selection with ties broken toward the lower index.
//
// HISA keeps the top-m blocks by representative score and then the top-k
// tokens of the kept blocks (gptget.net summary, "Methodology"; Chinese
// summary, method details); the flat scan keeps the top-k of all visible
// tokens.  All three use this kernel, one CTA per row:
//
//   1. radix select on the 32-bit order-preserving score keys (four 8-bit
//      digit passes, per-warp histograms, warp-aggregated increments) finds
//      the exact k-th largest key T and how many keys equal to T are taken;
//   2. an ordered compaction (each warp owns a contiguous slot range; ballots
//      give in-warp ranks, a scan over warps gives offsets) writes the kept
//      slots in ascending slot order, taking keys == T lowest slot first.
// Slots are laid out in ascending token order, so the output is ascending in
// token index, followed by -1 padding.  Key 0 marks an empty (masked) slot.
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSmemKeys = 16384;   // rows up to this many slots are staged in shared memory

struct SelShared {
    uint32_t hist[kSelWarps][256];
    uint32_t tot[256];
    uint32_t warp_a[kSelWarps];
    uint32_t warp_b[kSelWarps];
    uint32_t warp_c[kSelWarps];
    uint32_t warp_d[kSelWarps];
    uint32_t bcast[4];
};

// Where a row's keys come from.
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

__device__ __forceinline__ uint32_t block_sum(uint32_t v, SelShared& sh) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) sh.warp_a[warp] = v;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < kSelWarps; ++w) t += sh.warp_a[w];
    __syncthreads();
    return t;
}

// Exact k-th largest key among the nonzero keys of [0, n) (n_valid > k).
// Returns T and the number of keys equal to T that belong to the top k.
__device__ void radix_threshold(const Keys& keys, int n, int k, SelShared& sh, uint32_t& T,
                                int& take_eq) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t prefix = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) sh.hist[warp][i] = 0;
        __syncwarp();
        for (int base = warp * 32; base < n; base += kSelThreads) {
            const int c = base + lane;
            const uint32_t x = c < n ? keys(c) : 0u;
            const bool act = x != 0u && (x & mask) == prefix;
            const uint32_t bin = act ? ((x >> shift) & 255u) : 256u;
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (act && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[warp][bin], __popc(peers));
        }
        __syncthreads();
        if (tid < 256) {
            uint32_t s = 0;
            for (int w = 0; w < kSelWarps; ++w) s += sh.hist[w][tid];
            sh.tot[tid] = s;
        }
        __syncthreads();
        if (warp == 0) {
            // lane L owns bins 255-8L .. 248-8L, highest first
            uint32_t loc[8], lsum = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                loc[q] = sh.tot[255 - 8 * lane - q];
                lsum += loc[q];
            }
            uint32_t incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - lsum;
            if (excl < static_cast<uint32_t>(krem) && static_cast<uint32_t>(krem) <= incl) {
                uint32_t run = excl;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (run + loc[q] >= static_cast<uint32_t>(krem)) {
                        sh.bcast[0] = 255u - 8u * lane - q;
                        sh.bcast[1] = static_cast<uint32_t>(krem) - run;
                        break;
                    }
                    run += loc[q];
                }
            }
        }
        __syncthreads();
        prefix |= sh.bcast[0] << shift;
        mask |= 0xFFu << shift;
        krem = static_cast<int>(sh.bcast[1]);
        __syncthreads();
    }
    T = prefix;
    take_eq = krem;
}

// Ordered compaction.  Keeps keys > T, plus the first `take_eq` keys == T in
// slot order (with T == 0 every nonzero key is kept).  Calls emit(pos, slot,
// key) with pos = rank among kept slots in slot order.  Returns the count.
template <class Emit>
__device__ int compact(const Keys& keys, int n, uint32_t T, int take_eq, SelShared& sh, Emit emit) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_warp = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int w0 = warp * per_warp;
    const int w1 = min(n, w0 + per_warp);
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
        uint32_t eq_before = 0, off = 0;
        for (int w = 0; w < kSelWarps; ++w) {
            const uint32_t e = sh.warp_b[w];
            const int room = take_eq - static_cast<int>(eq_before);
            const uint32_t take = room <= 0 ? 0u : (static_cast<uint32_t>(room) < e ? room : e);
            sh.warp_c[w] = eq_before;
            sh.warp_d[w] = off;
            eq_before += e;
            off += sh.warp_a[w] + take;
        }
        sh.bcast[2] = off;
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
    const int total = static_cast<int>(sh.bcast[2]);
    __syncthreads();
    return total;
}

template <bool SMEM>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectParams p) {
    extern __shared__ uint32_t staged[];
    __shared__ SelShared sh;
    const int row = blockIdx.x;
    const int tid = threadIdx.x;

    int n = 0, kk = p.k, b = 0, t = 0, nb = 0;
    Keys keys{nullptr, nullptr, nullptr};
    if (p.mode == kSelF32Rows) {
        n = p.n;
        keys.x = p.x + static_cast<size_t>(row) * p.n;
    } else {
        t = query_position(p.q_seq, p.q_pos, p.len, p.batch, p.cap, row, &b);
        if (t < 0) {
            if (tid == 0) set_status(p.status, HISA_DEV_BAD_QUERY);
            if (p.mode == kSelBlocks) {
                for (int r = tid; r < p.mm; r += kSelThreads) {
                    p.blocks[static_cast<size_t>(row) * p.mm + r] = -1;
                    if (p.blocks_out) p.blocks_out[static_cast<size_t>(row) * p.mm + r] = -1;
                }
                if (tid == 0) {
                    p.nblocks[row] = 0;
                    if (p.nblocks_out) p.nblocks_out[row] = 0;
                }
            } else {
                for (int r = tid; r < p.k; r += kSelThreads) {
                    p.idx[static_cast<size_t>(row) * p.k + r] = -1;
                    if (p.scores) p.scores[static_cast<size_t>(row) * p.k + r] = __int_as_float(0x7fc00000);
                }
            }
            return;
        }
        keys.g = p.keys + static_cast<size_t>(row) * p.ldk;
        if (p.mode == kSelBlocks) {
            nb = t / p.B + 1;
            n = nb - 1;          // every block but the own one competes
            kk = p.m - 1;        // for m - 1 places
        } else if (p.mode == kSelHisaTokens) {
            n = p.nblocks[row] * p.B;
        } else {
            n = t + 1;
        }
    }

    if (p.mode == kSelBlocks && nb <= p.m) {
        // every visible block is kept
        int32_t* out = p.blocks + static_cast<size_t>(row) * p.mm;
        for (int r = tid; r < p.mm; r += kSelThreads) {
            const int v = r < nb ? r : -1;
            out[r] = v;
            if (p.blocks_out) p.blocks_out[static_cast<size_t>(row) * p.mm + r] = v;
        }
        if (tid == 0) {
            p.nblocks[row] = nb;
            if (p.nblocks_out) p.nblocks_out[row] = nb;
        }
        return;
    }

    if (SMEM) {
        for (int c = tid; c < n; c += kSelThreads) staged[c] = keys(c);
        __syncthreads();
        keys.smem = staged;
    }

    uint32_t T = 0;
    int take_eq = 0;
    if (kk > 0) {
        uint32_t nvalid = 0;
        for (int c = tid; c < n; c += kSelThreads) nvalid += keys(c) != 0u;
        nvalid = block_sum(nvalid, sh);
        if (nvalid > static_cast<uint32_t>(kk)) radix_threshold(keys, n, kk, sh, T, take_eq);
    }

    if (p.mode == kSelBlocks) {
        int32_t* out = p.blocks + static_cast<size_t>(row) * p.mm;
        int32_t* dbg = p.blocks_out ? p.blocks_out + static_cast<size_t>(row) * p.mm : nullptr;
        int kept = 0;
        if (kk > 0)
            kept = compact(keys, n, T, take_eq, sh, [&](int pos, int c, uint32_t) {
                out[pos] = c;
                if (dbg) dbg[pos] = c;
            });
        __syncthreads();
        for (int r = kept + tid; r < p.mm; r += kSelThreads) {
            const int v = r == kept ? nb - 1 : -1;   // own block last (largest id)
            out[r] = v;
            if (dbg) dbg[r] = v;
        }
        if (tid == 0) {
            p.nblocks[row] = kept + 1;
            if (p.nblocks_out) p.nblocks_out[row] = kept + 1;
        }
        return;
    }

    int32_t* idx = p.idx + static_cast<size_t>(row) * p.k;
    float* sc = p.scores ? p.scores + static_cast<size_t>(row) * p.k : nullptr;
    const int32_t* blk = p.mode == kSelHisaTokens ? p.blocks + static_cast<size_t>(row) * p.mm : nullptr;
    const int Bsz = p.B;
    const int kept = compact(keys, n, T, take_eq, sh, [&](int pos, int c, uint32_t x) {
        idx[pos] = blk ? blk[c / Bsz] * Bsz + c % Bsz : c;
        if (sc) sc[pos] = key_score(x);
    });
    for (int r = kept + tid; r < p.k; r += kSelThreads) {
        idx[r] = -1;
        if (sc) sc[r] = __int_as_float(0x7fc00000);
    }
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, int max_n, cudaStream_t s) {
    if (p.rows <= 0) return cudaSuccess;
    if (max_n <= kSmemKeys) {
        const size_t smem = static_cast<size_t>(max_n > 0 ? max_n : 1) * sizeof(uint32_t);
        cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        select_kernel<true><<<p.rows, kSelThreads, smem, s>>>(p);
    } else {
        select_kernel<false><<<p.rows, kSelThreads, 0, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace hisa
