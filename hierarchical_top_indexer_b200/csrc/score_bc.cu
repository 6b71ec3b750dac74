// Block-centric token scoring, for query rows that share their keys (a
// prefill chunk: thousands of rows select blocks of the same sequence).
//
// Stage 2 of HISA scores every token of each row's kept blocks with the
// indexer (arXiv abstract, stage (2); gptget.net summary, "Methodology").
// Scored row by row (score.cu), every row that kept a block brings that
// block's 32 KiB key tile to the SM again, and each tcgen05.mma has only the
// row's heads as its N.  Here the work is turned around: a work unit is one
// kept block of one sequence and up to kBcUnitPairs (row, slot) pairs that
// kept it.  The block's key tile is loaded once per unit into shared memory
// as the A operand (M = 128 tokens), and the query heads of R = 256 / npad
// rows at a time are stacked as the B operand (N = 256), so every MMA is
// full width and a key tile serves many rows.  The epilogue forms
// sum_h w[row,h] * max(0, q[row,h] . k) for each (token, row) and writes each
// row's 128 score keys to its candidate slots r*B .. r*B + 127, where r is
// the block's place in the row's kept list: the layout the row-centric kernel
// writes, so the same top-k kernel follows.  Each score is the same
// bf16 x bf16 dot product accumulated in fp32 over the same K steps, then the
// same head sum, as in the row-centric kernel.
//
// The (row, slot) pairs come grouped by block from an inverted index of the
// block stage's kept lists, built by three small kernels: count (a rank per
// pair inside its block), scan (block offsets and the work units) and
// scatter.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps
// 2-9 epilogue (two warps per TMEM lane quadrant, each taking half of the 256
// accumulator columns).  Every mbarrier wait is bounded (HISA_DEV_TIMEOUT).
#include "hisa_kernels.cuh"

namespace hisa {

namespace {

constexpr int kBcThreads = 320;
constexpr int kBcTile = 128;            // tokens per key tile (B = 128)
constexpr int kBcN = 256;               // accumulator columns: R rows x npad heads
constexpr int kBcStages = 2;            // query-group stages
constexpr int kBcMeta = 4;              // metadata / weight slots (see the producer)
constexpr int kBcUnitPairs = 32;        // (row, slot) pairs per work unit at most
constexpr int kBcABytes = kBcTile * 256;        // one key tile: two 16 KiB K halves
constexpr int kBcBBytes = kBcN * 256;           // one query group: two 32 KiB K halves

struct BcLayout {
    uint32_t a, b, w, meta, bars, misc, total;
};

__host__ __device__ inline BcLayout bc_layout() {
    BcLayout L;
    uint32_t off = 0;
    L.a = off;
    off += 2 * kBcABytes;
    L.b = off;
    off += kBcStages * kBcBBytes;
    L.w = off;
    off += kBcMeta * kBcN * 4;              // R rows x npad weights per slot
    L.meta = off;
    off += kBcMeta * 8 * 16;                // up to 8 rows x {row, slot, t, block}
    L.bars = off;
    off += (2 + 2 + 2 * kBcStages + 2 + 2 + kBcMeta) * 8;
    L.misc = off;
    off += 16;
    L.total = off;
    return L;
}

__device__ __forceinline__ bool bc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

__device__ __forceinline__ float bc_head_sum(int npad, uint32_t taddr, const float* wv) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < npad; g += 32) {
        uint32_t r[32];
        tmem_ld16_nowait(taddr + g, r);
        tmem_ld16_nowait(taddr + g + 16, r + 16);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 32; h += 4) {
            const float4 w4 = *reinterpret_cast<const float4*>(wv + g + h);
            fma2(a[0], a[1], w4.x, w4.y, fmaxf(__uint_as_float(r[h]), 0.f), fmaxf(__uint_as_float(r[h + 1]), 0.f));
            fma2(a[2], a[3], w4.z, w4.w, fmaxf(__uint_as_float(r[h + 2]), 0.f), fmaxf(__uint_as_float(r[h + 3]), 0.f));
        }
    }
    return (a[0] + a[1]) + (a[2] + a[3]);
}

__global__ void __launch_bounds__(kBcThreads, 1)
    bc_score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                    const BcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const BcLayout L = bc_layout();
    uint8_t* sA = smem + L.a;
    uint8_t* sB = smem + L.b;
    float* sW = reinterpret_cast<float*>(smem + L.w);
    int4* sMeta = reinterpret_cast<int4*>(smem + L.meta);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* afull = bars;                    // key tile landed      [2]
    uint64_t* aempty = bars + 2;               // key tile consumed    [2]
    uint64_t* bfull = bars + 4;                // query group landed   [kBcStages]
    uint64_t* bempty = bfull + kBcStages;      // query group consumed [kBcStages]
    uint64_t* tfull = bempty + kBcStages;      // accumulator ready    [2]
    uint64_t* tempty = tfull + 2;              // accumulator drained  [2]
    uint64_t* mfull = tempty + 2;              // group metadata and weights landed [kBcMeta]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npad = p.npad;
    const int R = kBcN / npad;                 // rows per query group
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(afull + i, 1);
            mbar_init(aempty + i, 1);
            mbar_init(tfull + i, 1);
            mbar_init(tempty + i, 8);
        }
        for (int s = 0; s < kBcStages; ++s) {
            mbar_init(bfull + s, 1);
            mbar_init(bempty + s, 1);
        }
        for (int m = 0; m < kBcMeta; ++m) mbar_init(mfull + m, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_async_smem();
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&qmap);
    }
    // weight columns H .. npad - 1 of every row stay zero (the copies write
    // columns 0 .. H - 1 only, so the two never touch the same bytes)
    for (int i = threadIdx.x; i < kBcMeta * kBcN; i += kBcThreads)
        if (i % npad >= p.H) sW[i] = 0.f;
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kBcN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dependency_wait();
    grid_launch_dependents();

    const int n_units = *p.n_units;
    const int u0 = static_cast<int>(static_cast<long long>(n_units) * blockIdx.x / gridDim.x);
    const int u1 = static_cast<int>(static_cast<long long>(n_units) * (blockIdx.x + 1) / gridDim.x);

    if (warp == 0) {
        const uint64_t keep = policy_evict_last();   // keys and queries are read again and again
        bool ok = true;
        int ua = 0, gq = 0;
        for (int u = u0; u < u1 && ok; ++u, ++ua) {
            // the unit, its pairs and their rows' positions, loaded by the warp
            const int4 ud = p.units[u];
            const int bj = ud.x, p0 = ud.y, np = ud.z;
            const int b = bj / p.nblk, j = bj - b * p.nblk;
            int row = 0, slot = 0, t = -1;
            if (lane < np) {
                const uint32_t pr = p.pairs[p0 + lane];
                row = static_cast<int>(pr >> 11);
                slot = static_cast<int>(pr & 2047u);
                t = p.plan[row].y;
            }
            const int row0 = __shfl_sync(0xffffffffu, row, 0);
            if (lane == 0) {
                if (!mbar_wait(aempty + (ua & 1), ((ua >> 1) & 1) ^ 1, abort_flag)) ok = false;
                if (ok) {
                    mbar_arrive_expect_tx(afull + (ua & 1), kBcABytes);
                    const int krow = b * p.cap + j * kBcTile;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
                        tma_load_2d_hint(sA + (ua & 1) * kBcABytes + kh * (kBcTile * 128), &kmap,
                                         afull + (ua & 1), kh * 64, krow, keep);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            const int ng = (np + R - 1) / R;
            for (int g = 0; g < ng && ok; ++g, ++gq) {
                const int s = gq % kBcStages, m = gq % kBcMeta;
                // The slot's previous group (gq - kBcStages) was consumed by
                // the MMA; its metadata slot (gq - kBcMeta) was read by the
                // epilogue, because the MMA of group gq - kBcStages needed its
                // accumulator back from group gq - kBcMeta.
                if (!bc_wait(bempty + s, ((gq / kBcStages) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                int4* md = sMeta + m * 8;
                int nvalid = 0;
                for (int q = 0; q < R; ++q) {
                    const int idx = g * R + q;
                    const int rq = __shfl_sync(0xffffffffu, row, idx < np ? idx : 0);
                    const int sq = __shfl_sync(0xffffffffu, slot, idx < np ? idx : 0);
                    const int tq = __shfl_sync(0xffffffffu, t, idx < np ? idx : 0);
                    if (lane == 0) md[q] = idx < np ? make_int4(rq, sq, tq, j) : make_int4(-1, 0, -1, j);
                    nvalid += idx < np;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(mfull + m, static_cast<uint32_t>(nvalid * p.H * 4));
                    for (int q = 0; q < nvalid; ++q)
                        bulk_load(sW + m * kBcN + q * npad, p.w + static_cast<size_t>(md[q].x) * p.H,
                                  static_cast<uint32_t>(p.H * 4), mfull + m);
                    mbar_arrive_expect_tx(bfull + s, kBcBBytes);
                    for (int q = 0; q < R; ++q) {
                        const int rq = q < nvalid ? md[q].x : row0;   // padding rows reuse a valid row
#pragma unroll
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_2d_hint(sB + s * kBcBBytes + kh * (kBcN * 128) + q * npad * 128, &qmap,
                                             bfull + s, kh * 64, rq * p.H, keep);
                    }
                }
                __syncwarp();
            }
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(p.status, HISA_DEV_TIMEOUT);
            }
            // after an abort no copy into this CTA's shared memory may still be
            // pending at exit (otherwise the consumers waited for every copy)
            if (!ok) {
                for (int n = gq > kBcStages ? gq - kBcStages : 0; n < gq; ++n)
                    mbar_wait(bfull + n % kBcStages, (n / kBcStages) & 1, nullptr);
                for (int n = gq > kBcMeta ? gq - kBcMeta : 0; n < gq; ++n)
                    mbar_wait(mfull + n % kBcMeta, (n / kBcMeta) & 1, nullptr);
                for (int n = ua > 2 ? ua - 2 : 0; n <= ua && n < u1 - u0; ++n)
                    mbar_wait(afull + (n & 1), (n >> 1) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kBcN);
            bool ok = true;
            int ua = 0, gq = 0;
            for (int u = u0; u < u1 && ok; ++u, ++ua) {
                const int np = p.units[u].z;
                const int ng = (np + R - 1) / R;
                if (!mbar_wait(afull + (ua & 1), (ua >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t a_base = smem_addr(sA + (ua & 1) * kBcABytes);
                for (int g = 0; g < ng; ++g, ++gq) {
                    const int s = gq % kBcStages, a = gq & 1;
                    if (!mbar_wait(bfull + s, (gq / kBcStages) & 1, abort_flag) ||
                        !mbar_wait(tempty + a, ((gq >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_base = smem_addr(sB + s * kBcBBytes);
                    const uint32_t d = tmem_base + static_cast<uint32_t>(a * kBcN);
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d, sw128_kmajor_desc(a_base + kh * (kBcTile * 128) + kk * 32),
                                      sw128_kmajor_desc(b_base + kh * (kBcN * 128) + kk * 32), idesc,
                                      (kh | kk) ? 1u : 0u);
                    umma_commit(bempty + s);
                    umma_commit(tfull + a);
                }
                if (!ok) break;
                umma_commit(aempty + (ua & 1));
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(p.status, HISA_DEV_TIMEOUT);
            }
            // every MMA of this CTA has finished before TMEM is released
            if (gq > 0) mbar_wait(tfull + ((gq - 1) & 1), ((gq - 1) >> 1) & 1, nullptr);
        }
    } else {
        const int quad = warp & 3;                 // TMEM lanes this warp reads
        const int half = (warp - 2) >> 2;          // accumulator columns [128 half, 128 half + 128)
        const int token = quad * 32 + lane;        // tile row = token in the block
        const int rpw = R / 2;                     // rows per warp
        bool ok = true;
        int gq = 0;
        for (int u = u0; u < u1 && ok; ++u) {
            const int np = p.units[u].z;
            const int ng = (np + R - 1) / R;
            for (int g = 0; g < ng; ++g, ++gq) {
                const int a = gq & 1, m = gq % kBcMeta;
                if (!bc_wait(tfull + a, (gq >> 1) & 1, abort_flag) ||
                    !bc_wait(mfull + m, (gq / kBcMeta) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int q = 0; q < rpw; ++q) {
                    const int pq = half * rpw + q;
                    const int4 md = sMeta[m * 8 + pq];
                    if (md.x < 0) continue;            // padding (uniform over the warp)
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                           static_cast<uint32_t>(a * kBcN + pq * npad);
                    const float acc = bc_head_sum(npad, taddr, sW + m * kBcN + pq * npad);
                    const int s = md.w * kBcTile + token;
                    // streamed past L2 (evict first), which keeps the keys and
                    // the queries that the next units read there
                    __stcs(p.out + static_cast<size_t>(md.x) * p.ldo + md.y * kBcTile + token,
                           s <= md.z ? score_key(acc) : 0u);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty + a);
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            set_status(p.status, HISA_DEV_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 2 * kBcN);
}

// ---------------------------------------------------------- the index

// One warp per row: each (row, r) pair of the row's kept list takes the next
// rank in its block's list.
__global__ void __launch_bounds__(256) bc_count_kernel(const BcParams p, const int32_t* blocks) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= p.n_q) return;
    const int4 pl = p.plan[row];
    if (pl.y < 0) return;
    for (int r = lane; r < pl.z; r += 32) {
        const int bj = pl.x * p.nblk + blocks[static_cast<size_t>(row) * p.mm + r];
        p.rank[static_cast<size_t>(row) * p.mm + r] = atomicAdd(p.cnt + bj, 1);
    }
    // work counters: the token slots this row scores (its kept blocks' tokens)
    if (p.counts && lane == 0)
        p.counts[static_cast<size_t>(row) * p.counts_ld + p.counts_col + 1] +=
            static_cast<unsigned long long>(pl.z) * kBcTile;
}

// One CTA: block offsets (exclusive scan of the counts) and the work units
// (each block's pairs in runs of at most kBcUnitPairs).
__global__ void __launch_bounds__(1024) bc_scan_kernel(const BcParams p, int nbj) {
    __shared__ uint32_t wp[32], wu[32];
    grid_dependency_wait();
    grid_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per = (nbj + 1023) / 1024;
    const int i0 = min(nbj, tid * per), i1 = min(nbj, i0 + per);
    uint32_t sp = 0, su = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t c = static_cast<uint32_t>(p.cnt[i]);
        sp += c;
        su += (c + kBcUnitPairs - 1) / kBcUnitPairs;
    }
    // exclusive scans of (pairs, units) over the threads
    uint32_t ip = sp, iu = su;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t a = __shfl_up_sync(0xffffffffu, ip, o), b = __shfl_up_sync(0xffffffffu, iu, o);
        if (lane >= o) {
            ip += a;
            iu += b;
        }
    }
    if (lane == 31) {
        wp[warp] = ip;
        wu[warp] = iu;
    }
    __syncthreads();
    uint32_t bp = 0, bu = 0, tu = 0;
    for (int w2 = 0; w2 < 32; ++w2) {
        bp += w2 < warp ? wp[w2] : 0u;
        bu += w2 < warp ? wu[w2] : 0u;
        tu += wu[w2];
    }
    uint32_t op = bp + ip - sp, ou = bu + iu - su;
    for (int i = i0; i < i1; ++i) {
        const int c = p.cnt[i];
        p.off[i] = static_cast<int>(op);
        for (int k = 0; k < c; k += kBcUnitPairs)
            p.units_w[ou++] = make_int4(i, static_cast<int>(op) + k, min(kBcUnitPairs, c - k), 0);
        op += static_cast<uint32_t>(c);
    }
    if (tid == 0) *p.n_units_w = static_cast<int>(tu);
}

// One warp per row: each pair to its place in its block's list.
__global__ void __launch_bounds__(256) bc_scatter_kernel(const BcParams p, const int32_t* blocks) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= p.n_q) return;
    const int4 pl = p.plan[row];
    if (pl.y < 0) return;
    for (int r = lane; r < pl.z; r += 32) {
        const size_t pr = static_cast<size_t>(row) * p.mm + r;
        const int bj = pl.x * p.nblk + blocks[pr];
        p.pairs_w[p.off[bj] + p.rank[pr]] = (static_cast<uint32_t>(row) << 11) | static_cast<uint32_t>(r);
    }
}

template <class K, class... A>
cudaError_t launch_pdl(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, A... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t bc_max_units(int n_q, int mm, int nbj) {
    return static_cast<size_t>(n_q) * mm / kBcUnitPairs + static_cast<size_t>(nbj);
}

cudaError_t launch_bc_index(const BcParams& p, const int32_t* blocks, int nbj, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(p.cnt, 0, sizeof(int32_t) * static_cast<size_t>(nbj), s);
    if (e != cudaSuccess) return e;
    const dim3 rows((p.n_q + 7) / 8);
    e = launch_pdl(bc_count_kernel, rows, dim3(256), 0, s, p, blocks);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bc_scan_kernel, dim3(1), dim3(1024), 0, s, p, nbj);
    if (e != cudaSuccess) return e;
    return launch_pdl(bc_scatter_kernel, rows, dim3(256), 0, s, p, blocks);
}

cudaError_t launch_bc_score(const CUtensorMap& kmap, const CUtensorMap& qmap, const BcParams& p, int sms,
                            cudaStream_t s) {
    const BcLayout L = bc_layout();
    if ((L.a | L.b) & 1023u) return cudaErrorInvalidValue;
    const size_t smem = L.total + 1024;
    const cudaError_t e = smem_limit(reinterpret_cast<const void*>(bc_score_kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bc_score_kernel, dim3(static_cast<unsigned>(sms)), dim3(kBcThreads), smem, s, kmap, qmap,
                      p);
}

}  // namespace hisa
