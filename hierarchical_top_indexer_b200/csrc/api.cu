// C ABI of the HISA indexer (include/hisa.h): argument checks, workspace
// layout, TMA tensor maps and kernel launches.  No allocation happens here:
// every buffer belongs to the caller, and so does the scratch space, except
// for hisa_select_static, whose scratch is one fixed device array below.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "hisa_kernels.cuh"

using namespace hisa;

namespace {

// ------------------------------------------------------------- driver API

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows, cols] with boxes of [box_rows, box_cols].
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, size_t elem, uint64_t rows,
              uint64_t cols, uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * elem};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The block representatives as a 3-D tensor [batch, nblk, 2d] bf16 with
// boxes of [1, 128, 64]: a box that runs past a sequence's nblk rows is
// zero-filled there instead of reading the next sequence's rows.
// boxes of `rows` representatives (128: a tile; bf: the children of one
// kept unit in a gathered level of the multi-level search)
bool pooled_map(CUtensorMap* map, const KvView& v, int rows = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(2 * v.d), static_cast<cuuint64_t>(v.nblk),
                                static_cast<cuuint64_t>(v.batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(2 * v.d) * 2,
                                   static_cast<cuuint64_t>(v.nblk) * 2 * v.d * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v.pooled_hl, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------- phase profiling

struct PhaseEvents {
    cudaEvent_t start, stop;
    int phase;
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<PhaseEvents> pending;   // recorded since the last read
    std::vector<cudaEvent_t> spare;     // reusable events

    cudaEvent_t take() {
        if (!spare.empty()) {
            cudaEvent_t e = spare.back();
            spare.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
};

Profiler& profiler() {
    static Profiler p;
    return p;
}

// Records an event pair around one kernel launch while profiling is on.
struct PhaseScope {
    int phase;
    cudaStream_t s;
    cudaEvent_t stop = nullptr;
    PhaseScope(int ph, cudaStream_t st) : phase(ph), s(st) {
        Profiler& P = profiler();
        std::lock_guard<std::mutex> g(P.mu);
        if (!P.on) return;
        cudaEvent_t start = P.take();
        stop = P.take();
        if (!start || !stop) {
            stop = nullptr;
            return;
        }
        record(start);
        P.pending.push_back({start, stop, phase});
    }
    ~PhaseScope() {
        if (stop) record(stop);
    }
    // while the stream is captured into a CUDA graph the pair becomes event
    // record nodes of the graph, timed each time the graph runs
    void record(cudaEvent_t e) const {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
            cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
        else
            cudaEventRecord(e, s);
    }
};

// SMs of the current device (looked up once per device).
int sm_count() {
    constexpr int kDevs = 64;
    static std::atomic<int> cached[kDevs];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kDevs && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < kDevs) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// ------------------------------------------------------------- validation

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_kv(const hisa_kv* kv, KvView* v) {
    if (!kv || !kv->keys || !kv->pooled || !kv->pooled_hl || !kv->len) return HISA_E_INVAL;
    if (kv->batch < 1 || kv->cap < 1 || kv->B < 1) return HISA_E_INVAL;
    if (kv->dtype != HISA_KEY_BF16 && kv->dtype != HISA_KEY_E4M3) return HISA_E_INVAL;
    if (kv->d != 64 && kv->d != 128) return HISA_E_UNSUPPORTED;
    if (kv->pool != HISA_POOL_MEAN && kv->pool != HISA_POOL_MAX) return HISA_E_INVAL;
    const bool e4m3 = kv->dtype == HISA_KEY_E4M3;
    if (e4m3 && !kv->key_scale) return HISA_E_INVAL;
    if (!aligned(kv->keys, 16) || !aligned(kv->pooled, 16) || !aligned(kv->pooled_hl, 16) ||
        !aligned(kv->len, 4) || (kv->key_scale && !aligned(kv->key_scale, 4)) ||
        (kv->status && !aligned(kv->status, 4)))
        return HISA_E_INVAL;
    if (static_cast<long long>(kv->batch) * kv->cap > INT_MAX) return HISA_E_UNSUPPORTED;
    v->keys = kv->keys;
    v->key_scale = kv->key_scale;
    v->pooled = kv->pooled;
    v->pooled_hl = kv->pooled_hl;
    v->len = kv->len;
    v->status = kv->status;
    v->batch = kv->batch;
    v->cap = kv->cap;
    v->d = kv->d;
    v->B = kv->B;
    v->nblk = (kv->cap + kv->B - 1) / kv->B;
    v->e4m3 = e4m3;
    v->pool_max = kv->pool == HISA_POOL_MAX;
    return HISA_OK;
}

bool select_block_size_ok(int B) {
    if (B == 8 || B == 16 || B == 32 || B == 64) return true;
    return B >= 128 && B <= 1024 && B % 128 == 0;
}

int check_queries(const uint16_t* Q, const float* w, const int32_t* q_seq, int n_q, int H, int k,
                  const int32_t* idx) {
    if (n_q < 0 || k < 1) return HISA_E_INVAL;
    if (H < 1 || H > 128) return HISA_E_UNSUPPORTED;
    if (n_q == 0) return HISA_OK;
    if (!Q || !w || !q_seq || !idx) return HISA_E_INVAL;
    if (!aligned(Q, 16) || !aligned(w, 4) || !aligned(q_seq, 4) || !aligned(idx, 4))
        return HISA_E_INVAL;
    return HISA_OK;
}

int npad_of(int H) { return (H + 15) / 16 * 16; }

// Workspace carving: consecutive 256-byte aligned regions.
struct Carve {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    }
};

struct HisaWs {
    size_t bkeys, blocks, nblocks, plan, tkeys, q8, w8, total;
    int ldb, ldt, mm;
    // block-centric token scoring (rows sharing their keys): the inverted index
    bool bc;
    size_t bc_cnt, bc_off, bc_rank, bc_pairs, bc_units, bc_nunits;
};

// Rows that share their keys (many rows per sequence, as a prefill chunk)
// score their tokens block by block (score_bc.cu) where that kernel applies:
// bf16 keys, B = 128, npad in {32, 64, 128}, H % 4 == 0.
bool use_block_centric(const KvView& v, int n_q, int H, int mm) {
    const int npad = (H + 15) / 16 * 16;
    return !v.e4m3 && v.B == 128 && (npad == 32 || npad == 64 || npad == 128) && H % 4 == 0 &&
           mm <= 2048 && n_q >= 256 && n_q >= 16 * v.batch && n_q < (1 << 21);
}

// e4m3 keys with d = 128 are scored on the fp8 tensor cores against split
// query heads (launch_qsplit), which the workspace holds.
bool f8_keys(const KvView& v) { return v.e4m3 && v.d == 128; }

void take_q8(Carve& c, const KvView& v, int n_q, int H, size_t* q8, size_t* w8) {
    *q8 = *w8 = 0;
    if (!f8_keys(v)) return;
    *q8 = c.take(static_cast<size_t>(n_q) * 2 * npad_of(H) * 128);
    *w8 = c.take(static_cast<size_t>(n_q) * npad_of(H) * 4);
}

HisaWs hisa_ws(const KvView& v, int n_q, int H, int m) {
    HisaWs w;
    w.mm = m < v.nblk ? m : v.nblk;
    w.ldb = static_cast<int>(round_up(v.nblk, 128));
    w.ldt = static_cast<int>(round_up(static_cast<size_t>(w.mm) * v.B, 128));
    Carve c;
    w.bkeys = c.take(static_cast<size_t>(n_q) * w.ldb * 4);
    w.blocks = c.take(static_cast<size_t>(n_q) * w.mm * 4);
    w.nblocks = c.take(static_cast<size_t>(n_q) * 4);
    w.plan = c.take(static_cast<size_t>(n_q) * 16);
    w.tkeys = c.take(static_cast<size_t>(n_q) * w.ldt * 4);
    take_q8(c, v, n_q, H, &w.q8, &w.w8);
    w.bc = use_block_centric(v, n_q, H, w.mm);
    if (w.bc) {
        const size_t nbj = static_cast<size_t>(v.batch) * v.nblk;
        const size_t pairs = static_cast<size_t>(n_q) * w.mm;
        w.bc_cnt = c.take(nbj * 4);
        w.bc_off = c.take(nbj * 4);
        w.bc_rank = c.take(pairs * 4);
        w.bc_pairs = c.take(pairs * 4);
        w.bc_units = c.take(bc_max_units(n_q, w.mm, static_cast<int>(nbj)) * 16);
        w.bc_nunits = c.take(4);
    }
    w.total = c.off;
    return w;
}

size_t flat_ld(const KvView& v) { return round_up(v.cap, 128); }

// The CUDA error behind the calling thread's last HISA_E_CUDA.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return HISA_OK;
    g_last_cuda_error = e;
    return HISA_E_CUDA;
}

bool keys_map(CUtensorMap* map, const KvView& v, int box_rows) {
    const uint64_t rows = static_cast<uint64_t>(v.batch) * v.cap;
    if (f8_keys(v))   // one 128-byte row per key: the fp8 operand layout as loaded
        return make_map(map, v.keys, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, 128, box_rows, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (v.e4m3)
        return make_map(map, v.keys, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, v.d, box_rows, v.d,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    return make_map(map, v.keys, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, v.d, box_rows, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

bool query_map(CUtensorMap* map, const uint16_t* Q, int n_q, int H, int d) {
    return make_map(map, Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(n_q) * H, d,
                    npad_of(H), 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

ScoreParams score_params(const KvView& v, const float* w, const int32_t* q_seq, const int32_t* q_pos,
                         int n_q, int H) {
    ScoreParams p;
    std::memset(&p, 0, sizeof p);
    p.len = v.len;
    p.key_scale = v.key_scale;
    p.status = v.status;
    p.batch = v.batch;
    p.cap = v.cap;
    p.nblk = v.nblk;
    p.B = v.B;
    p.w = w;
    p.q_seq = q_seq;
    p.q_pos = q_pos;
    p.n_q = n_q;
    p.H = H;
    p.npad = npad_of(H);
    p.counts_ld = 2;
    // More rows than sequences: rows share keys (a prefill chunk), which then
    // stay in L2; otherwise every row streams its own keys from HBM.
    p.keep_keys = n_q > v.batch ? 1 : 0;
    return p;
}

// Grid: one (or two) CTAs per SM at most, each taking an equal contiguous
// range of the row-major (row, tile) slots.
int run_score(int mode, const KvView& v, const CUtensorMap& amap, const CUtensorMap& qmap,
              ScoreParams& p, cudaStream_t s) {
    const bool e4m3 = mode != kScoreBlocks && v.e4m3;
    const int per_sm = score_config(mode, e4m3, v.d, p.npad, &p.stages, &p.stages8, &p.nacc);
    if (p.stages < 2 || p.nacc < 1) return HISA_E_UNSUPPORTED;
    p.total_tiles = static_cast<long long>(p.n_q) * p.tiles_per_row;
    if (p.total_tiles == 0) return HISA_OK;
    const int sms = sm_count();
    if (sms <= 0) return HISA_E_CUDA;
    // with the block selection fused in, whole rows per CTA
    const long long units = p.fuse ? p.n_q : p.total_tiles;
    const long long slots = static_cast<long long>(per_sm) * sms;
    const int grid = static_cast<int>(units < slots ? units : slots);
    const int phase = mode == kScoreBlocks ? HISA_PHASE_BLOCK_SCORE
                      : mode == kScoreFlat ? HISA_PHASE_FLAT_SCORE
                                           : HISA_PHASE_TOKEN_SCORE;
    PhaseScope ps(phase, s);
    return cuda_status(launch_score(mode, e4m3, v.d, amap, qmap, p, grid, s));
}

// fp8 scoring of e4m3 keys (d = 128): the query heads split into the
// workspace (launch_qsplit; already done by the caller when split = false),
// and the query tensor map and the weights aimed at them.
int split_queries(const KvView& v, const uint16_t* Q, const float* w, int n_q, int H, uint8_t* q8, float* w8,
                  cudaStream_t s) {
    if (!f8_keys(v)) return HISA_OK;
    PhaseScope ps(HISA_PHASE_QSPLIT, s);
    return cuda_status(launch_qsplit(Q, w, n_q, H, npad_of(H), q8, w8, s));
}

int prep_f8(const KvView& v, const uint16_t* Q, const float* w, int n_q, int H, uint8_t* q8, float* w8,
            CUtensorMap* qmap, ScoreParams& p, cudaStream_t s, bool split = true) {
    if (!f8_keys(v)) return HISA_OK;
    const int npad = npad_of(H);
    if (split) {
        const int rc = split_queries(v, Q, w, n_q, H, q8, w8, s);
        if (rc) return rc;
    }
    if (!make_map(qmap, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(n_q) * 2 * npad, 128,
                  2 * npad, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return HISA_E_CUDA;
    p.w8 = w8;
    p.scale_bulk = v.cap % 4 == 0 && aligned(v.key_scale, 16) ? 1 : 0;
    return HISA_OK;
}

// One block level: score the level's representatives (under the units kept
// one level up, if any) and keep each row's own block plus the best m - 1
// others into blocks [n_q, mm] / nblocks / plan.
struct BlockLevel {
    const KvView* v;
    int m, mm, ldb;
    uint32_t* bkeys;
    int32_t* blocks;
    int32_t* nblocks;
    int4* plan;
    int32_t* blocks_out;
    int32_t* nblocks_out;
    const int32_t* parent;   // kept superblocks [n_q, parent_ld] or null
    int parent_ld, bf;
    // gathered (the caller checked gathered_level()): score only the kept
    // superblocks' children; parent_n = the kept superblocks per row
    const int32_t* parent_n;
    int counts_col;
    // the decode step: row b is sequence b, whose new key the append kernel
    // launched just before writes (the caller guarantees the conditions of
    // the one-CTA-per-row block stage)
    int app;
};

int block_stage(const BlockLevel& lv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                const int32_t* q_pos, int n_q, int H, int k, uint64_t* counts, int counts_ld,
                cudaStream_t s) {
    const KvView& v = *lv.v;
    CUtensorMap pmap, qmap;
    if (!pooled_map(&pmap, v, lv.parent_n ? lv.bf : 128) || !query_map(&qmap, Q, n_q, H, v.d)) return HISA_E_CUDA;
    const int sms = sm_count();
    ScoreParams p = score_params(v, w, q_seq, q_pos, n_q, H);
    p.out = lv.bkeys;
    p.ldo = lv.ldb;
    p.tiles_per_row = lv.parent_n ? (lv.parent_ld * lv.bf + 127) / 128 : lv.ldb / 128;
    p.counts = reinterpret_cast<unsigned long long*>(counts);
    p.counts_ld = counts_ld;
    p.counts_col = lv.counts_col;
    p.parent = lv.parent;
    p.parent_ld = lv.parent_ld;
    p.bf = lv.bf;
    p.parent_n = lv.parent_n;
    // Short rows (up to kFuseMaxBlocks = 4 tiles of blocks) and at most two rows per SM: the
    // scoring kernel keeps the blocks itself, one CTA per row, which saves the
    // selection launch.  Longer rows score faster spread over every SM, and
    // many rows select faster in the selection kernel's one-CTA-per-row grid.
    const bool fuse = lv.parent_n ? true : lv.ldb <= kFuseMaxBlocks && n_q <= 2 * sms;
    if (lv.app) {
        if (!fuse) return HISA_E_UNSUPPORTED;
        p.app = 1;
        p.len_w = v.len;
    }
    if (fuse) {
        p.fuse = 1;
        p.m = lv.m;
        p.mm = lv.mm;
        p.sel_blocks = lv.blocks;
        p.sel_nblocks = lv.nblocks;
        p.sel_plan = lv.plan;
        p.sel_blocks_out = lv.blocks_out;
        p.sel_nblocks_out = lv.nblocks_out;
    }
    int rc = run_score(kScoreBlocks, v, pmap, qmap, p, s);
    if (rc || fuse) return rc;
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelBlocks;
    sp.keys = lv.bkeys;
    sp.ldk = lv.ldb;
    sp.rows = n_q;
    sp.k = k;
    sp.len = v.len;
    sp.q_seq = q_seq;
    sp.q_pos = q_pos;
    sp.status = v.status;
    sp.batch = v.batch;
    sp.cap = v.cap;
    sp.B = v.B;
    sp.m = lv.m;
    sp.mm = lv.mm;
    sp.blocks = lv.blocks;
    sp.nblocks = lv.nblocks;
    sp.plan = lv.plan;
    sp.blocks_out = lv.blocks_out;
    sp.nblocks_out = lv.nblocks_out;
    sp.tree = lv.parent ? 1 : 0;
    PhaseScope ps(HISA_PHASE_BLOCK_SELECT, s);
    return cuda_status(launch_select(sp, v.nblk, sms, s));
}

// Token level: score the kept blocks' tokens, keep the top k.
int token_stage(const KvView& v, const HisaWs& L, uint8_t* base, const uint16_t* Q, const float* w,
                const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int k, int32_t* idx,
                float* scores, uint64_t* counts, int counts_ld, int counts_col, int id_off,
                cudaStream_t s, bool split = true) {
    int32_t* blocks = reinterpret_cast<int32_t*>(base + L.blocks);
    int4* plan = reinterpret_cast<int4*>(base + L.plan);
    uint32_t* tkeys = reinterpret_cast<uint32_t*>(base + L.tkeys);
    CUtensorMap kmap, qmap;
    const int br = v.B < 128 ? v.B : 128;
    if (!keys_map(&kmap, v, br) || !query_map(&qmap, Q, n_q, H, v.d)) return HISA_E_CUDA;
    ScoreParams p = score_params(v, w, q_seq, q_pos, n_q, H);
    p.counts = reinterpret_cast<unsigned long long*>(counts);
    p.counts_ld = counts_ld;
    p.counts_col = counts_col;
    int rc = prep_f8(v, Q, w, n_q, H, base + L.q8, reinterpret_cast<float*>(base + L.w8), &qmap, p, s, split);
    if (rc) return rc;
    p.out = tkeys;
    p.ldo = L.ldt;
    p.tiles_per_row = L.ldt / 128;
    p.blocks = blocks;
    p.plan_in = plan;
    p.mm = L.mm;
    if (L.bc && id_off == 0) {
        // block-centric: an inverted index of the kept lists, then one unit
        // per (block, up to 32 rows that kept it)
        BcParams bp;
        std::memset(&bp, 0, sizeof bp);
        bp.plan = plan;
        bp.w = w;
        bp.n_q = n_q;
        bp.H = H;
        bp.npad = npad_of(H);
        bp.cap = v.cap;
        bp.nblk = v.nblk;
        bp.mm = L.mm;
        bp.cnt = reinterpret_cast<int32_t*>(base + L.bc_cnt);
        bp.off = reinterpret_cast<int32_t*>(base + L.bc_off);
        bp.rank = reinterpret_cast<int32_t*>(base + L.bc_rank);
        bp.pairs_w = reinterpret_cast<uint32_t*>(base + L.bc_pairs);
        bp.units_w = reinterpret_cast<int4*>(base + L.bc_units);
        bp.n_units_w = reinterpret_cast<int32_t*>(base + L.bc_nunits);
        bp.pairs = bp.pairs_w;
        bp.units = bp.units_w;
        bp.n_units = bp.n_units_w;
        bp.out = tkeys;
        bp.ldo = L.ldt;
        bp.status = v.status;
        bp.counts = reinterpret_cast<unsigned long long*>(counts);
        bp.counts_ld = counts_ld;
        bp.counts_col = counts_col;
        const int sms = sm_count();
        if (sms <= 0) return HISA_E_CUDA;
        PhaseScope ps(HISA_PHASE_TOKEN_SCORE, s);
        rc = cuda_status(launch_bc_index(bp, blocks, v.batch * v.nblk, s));
        if (rc) return rc;
        rc = cuda_status(launch_bc_score(kmap, qmap, bp, sms, s));
        if (rc) return rc;
    } else {
        rc = run_score(kScoreHisa, v, kmap, qmap, p, s);
        if (rc) return rc;
    }
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelHisaTokens;
    sp.keys = tkeys;
    sp.ldk = L.ldt;
    sp.rows = n_q;
    sp.k = k;
    sp.len = v.len;
    sp.q_seq = q_seq;
    sp.q_pos = q_pos;
    sp.status = v.status;
    sp.batch = v.batch;
    sp.cap = v.cap;
    sp.B = v.B;
    sp.mm = L.mm;
    sp.blocks = blocks;
    sp.plan = plan;
    sp.idx = idx;
    sp.scores = scores;
    sp.id_off = id_off;
    PhaseScope ps(HISA_PHASE_TOKEN_SELECT, s);
    return cuda_status(launch_select(sp, L.mm * v.B, sm_count(), s));
}

// The two stages on validated arguments (q_seq NULL: row i is sequence i).
int select_stages(const KvView& v, const HisaWs& L, uint8_t* base, const uint16_t* Q, const float* w,
                  const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx,
                  float* scores, int32_t* blocks_out, int32_t* nblocks_out, uint64_t* counts,
                  cudaStream_t s) {
    int rc;
    if (counts && cudaMemsetAsync(counts, 0, sizeof(uint64_t) * 2 * n_q, s) != cudaSuccess)
        return HISA_E_CUDA;
    // fp8 keys: the query split depends on the inputs alone, so it goes first
    // rather than between the two stages
    rc = split_queries(v, Q, w, n_q, H, base + L.q8, reinterpret_cast<float*>(base + L.w8), s);
    if (rc) return rc;
    BlockLevel lv;
    std::memset(&lv, 0, sizeof lv);
    lv.v = &v;
    lv.m = m;
    lv.mm = L.mm;
    lv.ldb = L.ldb;
    lv.bkeys = reinterpret_cast<uint32_t*>(base + L.bkeys);
    lv.blocks = reinterpret_cast<int32_t*>(base + L.blocks);
    lv.nblocks = reinterpret_cast<int32_t*>(base + L.nblocks);
    lv.plan = reinterpret_cast<int4*>(base + L.plan);
    lv.blocks_out = blocks_out;
    lv.nblocks_out = nblocks_out;
    rc = block_stage(lv, Q, w, q_seq, q_pos, n_q, H, k, counts, 2, s);
    if (rc) return rc;
    return token_stage(v, L, base, Q, w, q_seq, q_pos, n_q, H, k, idx, scores, counts, 2, 0, 0, s, false);
}

int hisa_select_impl(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                     const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx, float* scores,
                     int32_t* blocks_out, int32_t* nblocks_out, uint64_t* counts, void* ws,
                     size_t ws_bytes, cudaStream_t s) {
    KvView v;
    int rc = check_kv(kv, &v);
    if (rc) return rc;
    if (!select_block_size_ok(v.B)) return HISA_E_UNSUPPORTED;
    if (m < 1) return HISA_E_INVAL;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    const HisaWs L = hisa_ws(v, n_q, H, m);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HISA_E_WORKSPACE;
    return select_stages(v, L, static_cast<uint8_t*>(ws), Q, w, q_seq, q_pos, n_q, H, m, k, idx, scores,
                         blocks_out, nblocks_out, counts, s);
}

// Three-level search: a second index kv2 over the same keys with blocks of
// bf = kv2->B / kv->B first-level blocks (superblocks).
struct TreeWs {
    HisaWs L;            // first level and tokens
    size_t bkeys2, sblocks, nsblocks, plan2, total;
    int ldb2, ws;        // superblock score-key row length, kept superblocks per row
};

TreeWs tree_ws(const KvView& v, const KvView& v2, int n_q, int H, int W, int m) {
    TreeWs T;
    T.L = hisa_ws(v, n_q, H, m);
    T.ws = W < v2.nblk ? W : v2.nblk;
    T.ldb2 = static_cast<int>(round_up(v2.nblk, 128));
    Carve c;
    c.off = T.L.total;
    T.bkeys2 = c.take(static_cast<size_t>(n_q) * T.ldb2 * 4);
    T.sblocks = c.take(static_cast<size_t>(n_q) * T.ws * 4);
    T.nsblocks = c.take(static_cast<size_t>(n_q) * 4);
    T.plan2 = c.take(static_cast<size_t>(n_q) * 16);
    T.total = c.off;
    return T;
}

// kv2 must index the same keys as kv with a block size that is a multiple of kv's.
int check_tree(const hisa_kv* kv, const hisa_kv* kv2, KvView* v, KvView* v2) {
    int rc = check_kv(kv, v);
    if (rc) return rc;
    rc = check_kv(kv2, v2);
    if (rc) return rc;
    if (kv2->keys != kv->keys || kv2->key_scale != kv->key_scale || kv2->len != kv->len ||
        kv2->batch != kv->batch || kv2->cap != kv->cap || kv2->d != kv->d || kv2->dtype != kv->dtype ||
        kv2->pool != kv->pool || kv2->B % kv->B != 0)
        return HISA_E_INVAL;
    if (v2->nblk > kParentBits) return HISA_E_UNSUPPORTED;
    return HISA_OK;
}

// Search of any depth: level 0 (the block index) uses hisa_select's layout,
// each coarser level l a score-key row, a kept list, its lengths and a plan.
struct LevelsWs {
    HisaWs L;
    size_t bkeys[HISA_MAX_LEVELS], kept[HISA_MAX_LEVELS], nkept[HISA_MAX_LEVELS], plan[HISA_MAX_LEVELS];
    int ldb[HISA_MAX_LEVELS], mm[HISA_MAX_LEVELS];
    size_t total;
};

LevelsWs levels_ws(const KvView* v, int n, const int* keep, int n_q, int H) {
    LevelsWs T;
    std::memset(&T, 0, sizeof T);
    T.L = hisa_ws(v[0], n_q, H, keep[0]);
    T.mm[0] = T.L.mm;
    T.ldb[0] = T.L.ldb;
    Carve c;
    c.off = T.L.total;
    for (int l = 1; l < n; ++l) {
        T.mm[l] = keep[l] < v[l].nblk ? keep[l] : v[l].nblk;
        T.ldb[l] = static_cast<int>(round_up(v[l].nblk, 128));
        T.bkeys[l] = c.take(static_cast<size_t>(n_q) * T.ldb[l] * 4);
        T.kept[l] = c.take(static_cast<size_t>(n_q) * T.mm[l] * 4);
        T.nkept[l] = c.take(static_cast<size_t>(n_q) * 4);
        T.plan[l] = c.take(static_cast<size_t>(n_q) * 16);
    }
    T.total = c.off;
    return T;
}

// Every level indexes kv[0]'s keys; each unit size is a multiple of the one
// below; a level that parents another holds at most kParentBits units.
int check_levels(const hisa_kv* const* kv, int n, const int* keep, KvView* v) {
    if (!kv || !keep || n < 1 || n > HISA_MAX_LEVELS) return HISA_E_INVAL;
    for (int l = 0; l < n; ++l) {
        if (!kv[l] || keep[l] < 1) return HISA_E_INVAL;
        int rc = check_kv(kv[l], &v[l]);
        if (rc) return rc;
        if (l == 0) continue;
        const hisa_kv* a = kv[0];
        const hisa_kv* b = kv[l];
        if (b->keys != a->keys || b->key_scale != a->key_scale || b->len != a->len ||
            b->batch != a->batch || b->cap != a->cap || b->d != a->d || b->dtype != a->dtype ||
            b->pool != a->pool || b->B % kv[l - 1]->B != 0)
            return HISA_E_INVAL;
        if (v[l].nblk > kParentBits) return HISA_E_UNSUPPORTED;
    }
    return HISA_OK;
}

// Scratch of hisa_select_static: a file-scope device array, one per device
// (the runtime gives every device's context its own copy when it loads this
// module).  Its address is looked up once per device context and cached with
// that context's unique id, so a context re-created after a cudaDeviceReset
// gets a fresh lookup instead of a dangling address.
static __device__ __align__(256) uint8_t g_static_scratch[HISA_STATIC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context (0 if there is none yet).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

constexpr int kMaxDevices = 64;
struct StaticScratchSlot {
    unsigned long long ctx_id = 0;
    void* ptr = nullptr;
};
StaticScratchSlot g_static_scratch_slot[kMaxDevices];
std::mutex g_static_scratch_mu;

// Device address of the current device's copy of g_static_scratch.
int static_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HISA_E_CUDA;
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    StaticScratchSlot& slot = g_static_scratch_slot[dev];
    const unsigned long long id = current_ctx_id();
    if (id == 0 || id != slot.ctx_id || !slot.ptr) {
        void* p = nullptr;   // the lookup creates the context if there is none yet
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return HISA_E_CUDA;
        const unsigned long long now = current_ctx_id();
        if (now == 0) return HISA_E_CUDA;
        slot.ctx_id = now;
        slot.ptr = p;
    }
    *out = slot.ptr;
    return HISA_OK;
}

// A shard: global positions [tok_off, tok_off + cap) of every sequence, on
// block boundaries, with at most kRowKeys blocks (one selection CTA per row).
int check_cp(const hisa_kv* kv, int32_t tok_off, KvView* v) {
    const int rc = check_kv(kv, v);
    if (rc) return rc;
    if (!select_block_size_ok(v->B)) return HISA_E_UNSUPPORTED;
    if (tok_off < 0 || tok_off % v->B != 0 || v->cap % v->B != 0 ||
        static_cast<long long>(tok_off) + v->cap > 0x7fffffffLL)
        return HISA_E_INVAL;
    if (v->nblk > kRowKeys) return HISA_E_UNSUPPORTED;
    return HISA_OK;
}

// A level under kept units loads and scores only their children when that
// is at most a quarter of its blocks (otherwise scoring every block
// over all SMs and masking the others is as fast), a row's children fit one
// fused CTA (at most kFuseMaxBlocks), runs of bf children start on whole
// swizzle atoms (bf a power of two from 8 to 128) and there are at most two
// rows per SM.
bool gathered_level(int bf, int W, int nblk, int n_q) {
    const long long children = static_cast<long long>(W) * bf;
    return bf >= 8 && bf <= 128 && (bf & (bf - 1)) == 0 && W <= 256 && children <= kFuseMaxBlocks &&
           4 * children <= nblk && n_q <= 2 * sm_count();
}

}  // namespace

extern "C" {

int hisa_pool_blocks(const hisa_kv* kv, hisa_stream_t stream) {
    KvView v;
    const int rc = check_kv(kv, &v);
    if (rc) return rc;
    PhaseScope ps(HISA_PHASE_POOL, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status(launch_pool(v, reinterpret_cast<cudaStream_t>(stream)));
}

int hisa_append(const hisa_kv* kv, const void* tok, const float* tok_scale, hisa_stream_t stream) {
    KvView v;
    const int rc = check_kv(kv, &v);
    if (rc) return rc;
    if (!tok || !aligned(tok, 16)) return HISA_E_INVAL;
    if (v.e4m3 && (!tok_scale || !aligned(tok_scale, 4))) return HISA_E_INVAL;
    PhaseScope ps(HISA_PHASE_APPEND, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status(launch_append(v, tok, tok_scale, reinterpret_cast<cudaStream_t>(stream)));
}

size_t hisa_select_workspace_bytes(const hisa_kv* kv, int n_q, int H, int m, int k) {
    (void)k;
    KvView v;
    if (check_kv(kv, &v) || n_q < 0 || m < 1 || H < 1 || H > 128) return 0;
    return hisa_ws(v, n_q, H, m).total;
}

int hisa_select(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx, float* scores,
                void* ws, size_t ws_bytes, hisa_stream_t stream) {
    return hisa_select_impl(kv, Q, w, q_seq, q_pos, n_q, H, m, k, idx, scores, nullptr, nullptr,
                            nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int hisa_select_inspect(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                        const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx,
                        float* scores, int32_t* blocks, int32_t* nblocks, uint64_t* counts, void* ws,
                        size_t ws_bytes, hisa_stream_t stream) {
    return hisa_select_impl(kv, Q, w, q_seq, q_pos, n_q, H, m, k, idx, scores, blocks, nblocks,
                            counts, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t hisa_decode_step_workspace_bytes(const hisa_kv* kv, int H, int m, int k) {
    (void)k;
    KvView v;
    if (check_kv(kv, &v) || m < 1 || H < 1 || H > 128) return 0;
    return hisa_ws(v, v.batch, H, m).total;
}

int hisa_decode_step(const hisa_kv* kv, const void* tok, const float* tok_scale, const uint16_t* Q,
                     const float* w, int H, int m, int k, int32_t* idx, float* scores, void* ws,
                     size_t ws_bytes, hisa_stream_t stream) {
    KvView v;
    int rc = check_kv(kv, &v);
    if (rc) return rc;
    if (!select_block_size_ok(v.B)) return HISA_E_UNSUPPORTED;
    if (m < 1 || k < 1) return HISA_E_INVAL;
    if (H < 1 || H > 128) return HISA_E_UNSUPPORTED;
    if (!tok || !aligned(tok, 16) || (v.e4m3 && (!tok_scale || !aligned(tok_scale, 4)))) return HISA_E_INVAL;
    if (!Q || !w || !idx || !aligned(Q, 16) || !aligned(w, 4) || !aligned(idx, 4) ||
        (scores && !aligned(scores, 4)))
        return HISA_E_INVAL;
    const int n_q = v.batch;
    const HisaWs L = hisa_ws(v, n_q, H, m);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    const int sms = sm_count();
    if (sms <= 0) return HISA_E_CUDA;
    if (L.ldb > kFuseMaxBlocks || n_q > 2 * sms) {
        // rows too long (or too many) for one CTA per row: the append and the
        // selection as separate launches, with the same results
        {
            PhaseScope ps(HISA_PHASE_APPEND, s);
            rc = cuda_status(launch_append(v, tok, tok_scale, s));
            if (rc) return rc;
        }
        return select_stages(v, L, base, Q, w, nullptr, nullptr, n_q, H, m, k, idx, scores, nullptr,
                             nullptr, nullptr, s);
    }
    BlockLevel lv;
    std::memset(&lv, 0, sizeof lv);
    lv.v = &v;
    lv.m = m;
    lv.mm = L.mm;
    lv.ldb = L.ldb;
    lv.bkeys = reinterpret_cast<uint32_t*>(base + L.bkeys);
    lv.blocks = reinterpret_cast<int32_t*>(base + L.blocks);
    lv.nblocks = reinterpret_cast<int32_t*>(base + L.nblocks);
    lv.plan = reinterpret_cast<int4*>(base + L.plan);
    lv.app = 1;
    rc = split_queries(v, Q, w, n_q, H, base + L.q8, reinterpret_cast<float*>(base + L.w8), s);
    if (rc) return rc;
    {
        // the append, which the block scoring does not wait for (see
        // ScoreParams::app); it goes right before that kernel
        PhaseScope ps(HISA_PHASE_APPEND, s);
        rc = cuda_status(launch_append(v, tok, tok_scale, s, true));
        if (rc) return rc;
    }
    rc = block_stage(lv, Q, w, nullptr, nullptr, n_q, H, k, nullptr, 2, s);
    if (rc) return rc;
    return token_stage(v, L, base, Q, w, nullptr, nullptr, n_q, H, k, idx, scores, nullptr, 2, 0, 0, s, false);
}

int hisa_select_static(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                       const int32_t* q_pos, int n_q, int H, int m, int k, int32_t* idx,
                       float* scores, hisa_stream_t stream) {
    KvView v;
    int rc = check_kv(kv, &v);
    if (rc) return rc;
    if (!select_block_size_ok(v.B)) return HISA_E_UNSUPPORTED;
    if (m < 1) return HISA_E_INVAL;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    const size_t need = hisa_ws(v, n_q, H, m).total;
    if (need > HISA_STATIC_SCRATCH_BYTES) return HISA_E_SCRATCH_LIMIT;
    void* ws = nullptr;
    rc = static_scratch(&ws);
    if (rc) return rc;
    return hisa_select_impl(kv, Q, w, q_seq, q_pos, n_q, H, m, k, idx, scores, nullptr, nullptr,
                            nullptr, ws, HISA_STATIC_SCRATCH_BYTES,
                            reinterpret_cast<cudaStream_t>(stream));
}

// Flat scan workspace: score keys [n_q, round_up(cap, 128)], then (fp8
// scoring) the split query heads.
struct FlatWs {
    size_t keys, q8, w8, total;
};

FlatWs flat_ws(const KvView& v, int n_q, int H) {
    FlatWs f;
    Carve c;
    f.keys = c.take(static_cast<size_t>(n_q) * flat_ld(v) * 4);
    take_q8(c, v, n_q, H, &f.q8, &f.w8);
    f.total = c.off;
    return f;
}

size_t hisa_tree_workspace_bytes(const hisa_kv* kv, const hisa_kv* kv2, int n_q, int H, int W, int m,
                                 int k) {
    (void)k;
    KvView v, v2;
    if (check_tree(kv, kv2, &v, &v2) || n_q < 0 || m < 1 || W < 1 || H < 1 || H > 128) return 0;
    return tree_ws(v, v2, n_q, H, W, m).total;
}

int hisa_tree_select(const hisa_kv* kv, const hisa_kv* kv2, const uint16_t* Q, const float* w,
                     const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int W, int m, int k,
                     int32_t* idx, float* scores, int32_t* sblocks, int32_t* nsblocks, int32_t* blocks,
                     int32_t* nblocks, uint64_t* counts, void* ws, size_t ws_bytes,
                     hisa_stream_t stream) {
    KvView v, v2;
    int rc = check_tree(kv, kv2, &v, &v2);
    if (rc) return rc;
    if (!select_block_size_ok(v.B)) return HISA_E_UNSUPPORTED;
    if (m < 1 || W < 1) return HISA_E_INVAL;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    const TreeWs T = tree_ws(v, v2, n_q, H, W, m);
    if (!ws || !aligned(ws, 256) || ws_bytes < T.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    if (counts && cudaMemsetAsync(counts, 0, sizeof(uint64_t) * 3 * n_q, s) != cudaSuccess)
        return HISA_E_CUDA;
    // level 2: superblocks, the own one plus the best W - 1
    BlockLevel l2;
    std::memset(&l2, 0, sizeof l2);
    l2.v = &v2;
    l2.m = W;
    l2.mm = T.ws;
    l2.ldb = T.ldb2;
    l2.bkeys = reinterpret_cast<uint32_t*>(base + T.bkeys2);
    l2.blocks = reinterpret_cast<int32_t*>(base + T.sblocks);
    l2.nblocks = reinterpret_cast<int32_t*>(base + T.nsblocks);
    l2.plan = reinterpret_cast<int4*>(base + T.plan2);
    l2.blocks_out = sblocks;
    l2.nblocks_out = nsblocks;
    rc = block_stage(l2, Q, w, q_seq, q_pos, n_q, H, k, counts, 3, s);
    if (rc) return rc;
    // level 1: the blocks under the kept superblocks, the own one plus the best m - 1
    BlockLevel l1;
    std::memset(&l1, 0, sizeof l1);
    l1.v = &v;
    l1.m = m;
    l1.mm = T.L.mm;
    l1.ldb = T.L.ldb;
    l1.bkeys = reinterpret_cast<uint32_t*>(base + T.L.bkeys);
    l1.blocks = reinterpret_cast<int32_t*>(base + T.L.blocks);
    l1.nblocks = reinterpret_cast<int32_t*>(base + T.L.nblocks);
    l1.plan = reinterpret_cast<int4*>(base + T.L.plan);
    l1.blocks_out = blocks;
    l1.nblocks_out = nblocks;
    l1.parent = l2.blocks;
    l1.parent_ld = T.ws;
    l1.bf = v2.B / v.B;
    l1.counts_col = 1;
    if (gathered_level(l1.bf, T.ws, v.nblk, n_q)) l1.parent_n = l2.nblocks;
    rc = block_stage(l1, Q, w, q_seq, q_pos, n_q, H, k, counts, 3, s);
    if (rc) return rc;
    return token_stage(v, T.L, base, Q, w, q_seq, q_pos, n_q, H, k, idx, scores, counts, 3, 1, 0, s);
}

size_t hisa_levels_workspace_bytes(const hisa_kv* const* kv, int n_levels, const int* keep, int n_q,
                                   int H, int k) {
    (void)k;
    KvView v[HISA_MAX_LEVELS];
    if (check_levels(kv, n_levels, keep, v) || n_q < 0 || H < 1 || H > 128) return 0;
    return levels_ws(v, n_levels, keep, n_q, H).total;
}

int hisa_levels_select(const hisa_kv* const* kv, int n_levels, const int* keep, const uint16_t* Q,
                       const float* w, const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int k,
                       int32_t* idx, float* scores, int32_t* const* kept, int32_t* const* nkept,
                       uint64_t* counts, void* ws, size_t ws_bytes, hisa_stream_t stream) {
    KvView v[HISA_MAX_LEVELS];
    int rc = check_levels(kv, n_levels, keep, v);
    if (rc) return rc;
    if (!select_block_size_ok(v[0].B)) return HISA_E_UNSUPPORTED;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    const LevelsWs T = levels_ws(v, n_levels, keep, n_q, H);
    if (!ws || !aligned(ws, 256) || ws_bytes < T.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    const int cld = n_levels + 1;   // counts: units scored per level, then token slots
    if (counts && cudaMemsetAsync(counts, 0, sizeof(uint64_t) * cld * n_q, s) != cudaSuccess)
        return HISA_E_CUDA;
    // from the coarsest level down: the own unit plus the best keep[l] - 1
    // candidates, the candidates below the top being the children of the
    // units kept one level up (gathered where gathered_level allows)
    const int32_t* parent = nullptr;
    const int32_t* parent_n = nullptr;
    int parent_ld = 0;
    for (int l = n_levels - 1; l >= 0; --l) {
        BlockLevel lv;
        std::memset(&lv, 0, sizeof lv);
        lv.v = &v[l];
        lv.m = keep[l];
        lv.mm = T.mm[l];
        lv.ldb = T.ldb[l];
        lv.bkeys = reinterpret_cast<uint32_t*>(base + (l ? T.bkeys[l] : T.L.bkeys));
        lv.blocks = reinterpret_cast<int32_t*>(base + (l ? T.kept[l] : T.L.blocks));
        lv.nblocks = reinterpret_cast<int32_t*>(base + (l ? T.nkept[l] : T.L.nblocks));
        lv.plan = reinterpret_cast<int4*>(base + (l ? T.plan[l] : T.L.plan));
        lv.blocks_out = kept ? kept[l] : nullptr;
        lv.nblocks_out = nkept ? nkept[l] : nullptr;
        lv.counts_col = l;
        if (parent) {
            lv.parent = parent;
            lv.parent_ld = parent_ld;
            lv.bf = v[l + 1].B / v[l].B;
            if (gathered_level(lv.bf, parent_ld, v[l].nblk, n_q)) lv.parent_n = parent_n;
        }
        rc = block_stage(lv, Q, w, q_seq, q_pos, n_q, H, k, counts, cld, s);
        if (rc) return rc;
        parent = lv.blocks;
        parent_n = lv.nblocks;
        parent_ld = lv.mm;
    }
    return token_stage(v[0], T.L, base, Q, w, q_seq, q_pos, n_q, H, k, idx, scores, counts, cld,
                       n_levels - 1, 0, s);
}

// ---------------------------------------------------- context parallelism

size_t hisa_cp_workspace_bytes(const hisa_kv* kv, int32_t tok_off, int n_q, int H, int m, int k) {
    (void)k;
    KvView v;
    if (check_cp(kv, tok_off, &v) || n_q < 0 || m < 1 || H < 1 || H > 128) return 0;
    return hisa_ws(v, n_q, H, m).total;
}

int hisa_cp_blocks(const hisa_kv* kv, int32_t tok_off, const uint16_t* Q, const float* w,
                   const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m, int32_t* cand_ids,
                   float* cand_scores, void* ws, size_t ws_bytes, hisa_stream_t stream) {
    KvView v;
    int rc = check_cp(kv, tok_off, &v);
    if (rc) return rc;
    if (m < 1) return HISA_E_INVAL;
    rc = check_queries(Q, w, q_seq, n_q, H, m, cand_ids);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    if (!q_pos || !cand_scores || !aligned(q_pos, 4) || !aligned(cand_scores, 4)) return HISA_E_INVAL;
    const HisaWs L = hisa_ws(v, n_q, H, m);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* bkeys = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.bkeys);
    CUtensorMap pmap, qmap;
    if (!pooled_map(&pmap, v) || !query_map(&qmap, Q, n_q, H, v.d)) return HISA_E_CUDA;
    // the shard's visible blocks scored into the workspace ...
    ScoreParams p = score_params(v, w, q_seq, q_pos, n_q, H);
    p.out = bkeys;
    p.ldo = L.ldb;
    p.tiles_per_row = L.ldb / 128;
    p.cp = 1;
    p.tok_off = tok_off;
    rc = run_score(kScoreBlocks, v, pmap, qmap, p, s);
    if (rc) return rc;
    // ... and the best m - 1 of them but the own block, then the own block
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelCpBlocks;
    sp.keys = bkeys;
    sp.ldk = L.ldb;
    sp.rows = n_q;
    sp.k = m;
    sp.m = m;
    sp.len = v.len;
    sp.q_seq = q_seq;
    sp.q_pos = q_pos;
    sp.status = v.status;
    sp.batch = v.batch;
    sp.cap = v.cap;
    sp.B = v.B;
    sp.id_off = tok_off / v.B;
    sp.idx = cand_ids;
    sp.scores = cand_scores;
    PhaseScope ps(HISA_PHASE_BLOCK_SELECT, s);
    return cuda_status(launch_select(sp, v.nblk, sm_count(), s));
}

int hisa_cp_tokens(const hisa_kv* kv, int32_t tok_off, const uint16_t* Q, const float* w,
                   const int32_t* q_seq, const int32_t* q_pos, int n_q, int H, int m, int k,
                   const int32_t* kept, int32_t* idx, float* scores, void* ws, size_t ws_bytes,
                   hisa_stream_t stream) {
    KvView v;
    int rc = check_cp(kv, tok_off, &v);
    if (rc) return rc;
    if (m < 1) return HISA_E_INVAL;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    if (!q_pos || !kept || !aligned(q_pos, 4) || !aligned(kept, 4) || (scores && !aligned(scores, 4)))
        return HISA_E_INVAL;
    const HisaWs L = hisa_ws(v, n_q, H, m);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    CpLocalizeParams lp;
    std::memset(&lp, 0, sizeof lp);
    lp.kept = kept;
    lp.m = m;
    lp.q_seq = q_seq;
    lp.q_pos = q_pos;
    lp.len = v.len;
    lp.status = v.status;
    lp.batch = v.batch;
    lp.cap = v.cap;
    lp.B = v.B;
    lp.tok_off = tok_off;
    lp.rows = n_q;
    lp.mm = L.mm;
    lp.blocks = reinterpret_cast<int32_t*>(base + L.blocks);
    lp.nblocks = reinterpret_cast<int32_t*>(base + L.nblocks);
    lp.plan = reinterpret_cast<int4*>(base + L.plan);
    {
        PhaseScope ps(HISA_PHASE_BLOCK_SELECT, s);
        rc = cuda_status(launch_cp_localize(lp, s));
        if (rc) return rc;
    }
    return token_stage(v, L, base, Q, w, q_seq, q_pos, n_q, H, k, idx, scores, nullptr, 2, 0, tok_off, s);
}

int hisa_merge_topk(const int32_t* ids, const float* scores, int lists, int rows, int n, int k,
                    int32_t* idx, float* out_scores, hisa_stream_t stream) {
    if (lists < 1 || rows < 0 || n < 0 || k < 1) return HISA_E_INVAL;
    if (static_cast<long long>(lists) * n > kRowKeys) return HISA_E_UNSUPPORTED;
    if (rows == 0) return HISA_OK;
    if (!ids || !scores || !idx || !aligned(ids, 4) || !aligned(scores, 4) || !aligned(idx, 4) ||
        (out_scores && !aligned(out_scores, 4)))
        return HISA_E_INVAL;
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelMerge;
    sp.x = scores;
    sp.ids = ids;
    sp.lists = lists;
    sp.n = n;
    sp.rows = rows;
    sp.k = k;
    sp.idx = idx;
    sp.scores = out_scores;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    PhaseScope ps(HISA_PHASE_MERGE, s);
    return cuda_status(launch_select(sp, lists * n, sm_count(), s));
}

size_t hisa_sparse_attn_workspace_bytes(int n_q, int k) {
    if (n_q < 0 || k < 1) return 0;
    return attn_workspace_bytes(n_q, k);
}

int hisa_sparse_attn(const uint16_t* Qa, int Ha, const uint16_t* Kc, const uint16_t* Vc, const int32_t* len,
                     int batch, int cap, int d, const int32_t* q_seq, const int32_t* idx, int n_q, int k,
                     float scale, float* out, float* lse, uint32_t* status, void* ws, size_t ws_bytes,
                     hisa_stream_t stream) {
    if (n_q < 0 || k < 1 || batch < 1 || cap < 1 || !(scale > 0.f) || !std::isfinite(scale)) return HISA_E_INVAL;
    if (Ha < 1 || Ha > 128 || d != 128) return HISA_E_UNSUPPORTED;
    if (n_q == 0) return HISA_OK;
    if (!Qa || !Kc || !Vc || !len || !q_seq || !idx || !out || !status) return HISA_E_INVAL;
    if (!aligned(Qa, 16) || !aligned(Kc, 16) || !aligned(Vc, 16) || !aligned(out, 16) || !aligned(len, 4) ||
        !aligned(q_seq, 4) || !aligned(idx, 4) || !aligned(status, 4) || (lse && !aligned(lse, 4)))
        return HISA_E_INVAL;
    if (!ws || !aligned(ws, 256) || ws_bytes < attn_workspace_bytes(n_q, k)) return HISA_E_WORKSPACE;
    AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.q = Qa;
    p.kc = Kc;
    p.vc = Vc;
    p.idx = idx;
    p.q_seq = q_seq;
    p.len = len;
    p.batch = batch;
    p.cap = cap;
    p.n_q = n_q;
    p.Ha = Ha;
    p.k = k;
    p.T = (k + 127) / 128;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out = out;
    p.lse = lse;
    p.status = status;
    attn_carve(p, ws);
    const int sms = sm_count();
    if (sms <= 0) return HISA_E_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    PhaseScope ps(HISA_PHASE_ATTN, s);
    return cuda_status(launch_attn(p, sms, s));
}

int hisa_selftest_wait(uint32_t* status, hisa_stream_t stream) {
    if (!status || !aligned(status, 4)) return HISA_E_INVAL;
    return cuda_status(launch_wait_probe(status, reinterpret_cast<cudaStream_t>(stream)));
}

int hisa_pool_tail(const hisa_kv* kv, hisa_stream_t stream) {
    KvView v;
    const int rc = check_kv(kv, &v);
    if (rc) return rc;
    PhaseScope ps(HISA_PHASE_APPEND, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status(launch_pool_tail(v, reinterpret_cast<cudaStream_t>(stream)));
}

size_t dsa_flat_workspace_bytes(const hisa_kv* kv, int n_q, int H, int k) {
    (void)k;
    KvView v;
    if (check_kv(kv, &v) || n_q < 0 || H < 1 || H > 128) return 0;
    return flat_ws(v, n_q, H).total;
}

int dsa_flat_select(const hisa_kv* kv, const uint16_t* Q, const float* w, const int32_t* q_seq,
                    const int32_t* q_pos, int n_q, int H, int k, int32_t* idx, float* scores, void* ws,
                    size_t ws_bytes, hisa_stream_t stream) {
    KvView v;
    int rc = check_kv(kv, &v);
    if (rc) return rc;
    if (!select_block_size_ok(v.B)) return HISA_E_UNSUPPORTED;
    rc = check_queries(Q, w, q_seq, n_q, H, k, idx);
    if (rc) return rc;
    if (n_q == 0) return HISA_OK;
    const size_t ld = flat_ld(v);
    const FlatWs F = flat_ws(v, n_q, H);
    if (!ws || !aligned(ws, 256) || ws_bytes < F.total) return HISA_E_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    CUtensorMap kmap, qmap;
    if (!keys_map(&kmap, v, v.B < 128 ? v.B : 128) || !query_map(&qmap, Q, n_q, H, v.d))
        return HISA_E_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    uint32_t* keys = reinterpret_cast<uint32_t*>(base + F.keys);
    ScoreParams p = score_params(v, w, q_seq, q_pos, n_q, H);
    rc = prep_f8(v, Q, w, n_q, H, base + F.q8, reinterpret_cast<float*>(base + F.w8), &qmap, p, s);
    if (rc) return rc;
    p.out = keys;
    p.ldo = static_cast<int>(ld);
    p.tiles_per_row = static_cast<int>(ld / 128);
    rc = run_score(kScoreFlat, v, kmap, qmap, p, s);
    if (rc) return rc;
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelFlatTokens;
    sp.keys = keys;
    sp.ldk = static_cast<int>(ld);
    sp.rows = n_q;
    sp.k = k;
    sp.len = v.len;
    sp.q_seq = q_seq;
    sp.q_pos = q_pos;
    sp.status = v.status;
    sp.batch = v.batch;
    sp.cap = v.cap;
    sp.B = v.B;
    sp.idx = idx;
    sp.scores = scores;
    PhaseScope ps(HISA_PHASE_FLAT_SELECT, s);
    return cuda_status(launch_select(sp, v.cap, sm_count(), s));
}

int hisa_topk_f32(const float* x, int rows, int n, int k, int32_t* idx, hisa_stream_t stream) {
    if (rows < 0 || n < 0 || k < 1) return HISA_E_INVAL;
    if (rows == 0) return HISA_OK;
    if (!x || !idx || !aligned(x, 4) || !aligned(idx, 4)) return HISA_E_INVAL;
    SelectParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.mode = kSelF32Rows;
    sp.x = x;
    sp.n = n;
    sp.rows = rows;
    sp.k = k;
    sp.idx = idx;
    PhaseScope ps(HISA_PHASE_TOPK, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status(launch_select(sp, n, sm_count(), reinterpret_cast<cudaStream_t>(stream)));
}

int hisa_profile_enable(int on) {
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    P.on = on != 0;
    return HISA_OK;
}

int hisa_profile_read(float* ms, int* launches, int reset) {
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    if (ms)
        for (int i = 0; i < HISA_NUM_PHASES; ++i) ms[i] = 0.f;
    if (launches)
        for (int i = 0; i < HISA_NUM_PHASES; ++i) launches[i] = 0;
    int rc = HISA_OK;
    for (const PhaseEvents& e : P.pending) {
        float t = 0.f;
        if (cudaEventSynchronize(e.stop) != cudaSuccess || cudaEventElapsedTime(&t, e.start, e.stop) != cudaSuccess)
            rc = HISA_E_CUDA;
        if (ms) ms[e.phase] += t;
        if (launches) launches[e.phase] += 1;
    }
    if (reset) {
        for (const PhaseEvents& e : P.pending) {
            P.spare.push_back(e.start);
            P.spare.push_back(e.stop);
        }
        P.pending.clear();
    }
    return rc;
}

const char* hisa_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

const char* hisa_status_string(int code) {
    switch (code) {
        case HISA_OK: return "ok";
        case HISA_E_INVAL: return "invalid argument";
        case HISA_E_UNSUPPORTED: return "unsupported size";
        case HISA_E_WORKSPACE: return "workspace too small or misaligned";
        case HISA_E_CUDA: return "CUDA error";
        case HISA_E_SCRATCH_LIMIT: return "call needs more than HISA_STATIC_SCRATCH_BYTES of scratch";
        default: return "unknown status";
    }
}

}  // extern "C"
