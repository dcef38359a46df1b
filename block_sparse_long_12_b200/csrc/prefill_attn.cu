// Step 2 of MSA for a causal prefill chunk on the tensor cores: every query
// head attends over its group's selected blocks of the real K/V.
//
// Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 2: the heads of
// a group share one block list, so one KV block serves all of them (Q1/Q2/Q3
// -> I1, Q4/Q5/Q6 -> I2).  In prefill every token has its own list, and the
// lists of neighbouring tokens need not overlap, so the work is organised by
// block instead of by token: every (row, selected block) pair is put in the
// bucket of its block, and a tile is up to 128 / r member rows of one bucket
// with their r heads (M = 128) against that one block.  A pair's attention is
// then exact within the block -- S = Q K^T, softmax over the block's visible
// keys, O = P V normalised by the block's sum -- and its output and log2 sum
// (bf16) go to the workspace; a merge kernel combines each row's k pairs by
// log-sum-exp into the row's output.  No tile computes a row that did not
// select its block.
//
// Per pass over up to prefill_rows_per_pass(k) query rows:
//   pa_count_kernel     pairs per bucket and each pair's rank in it;
//   pa_tilecount_kernel pairs and tiles per scan block of 1024 buckets;
//   pa_emit_kernel      bucket offsets and the tile list (bucket order);
//   pa_scatter_kernel   members grouped by bucket;
//   pa_tile_kernel      the tiles, persistent, one contiguous range per SM:
//     warp 3      stages each tile's descriptor and member list in a
//                 shared-memory ring that every other role reads;
//     warp 0      TMA of the block's K and V tiles (2-stage ring, reloaded
//                 only when the bucket changes);
//     warp 1      TMEM owner, issues tcgen05.mma: S = Q K^T (M 128, N Bk)
//                 into a double-buffered S buffer, and O = P V (N = D) with P
//                 read from TMEM (it overwrites its own S buffer) into a
//                 double-buffered O;
//     warp 2      TMA gather of the members' query rows (one box of the r
//                 heads per member and 64-dim half, 2-stage ring);
//     warps 4-11  softmax, two warps per TMEM lane quadrant on half of the
//                 block's keys each: mask keys after the row, row max
//                 (exchanged between the two), P = 2^(z*c - m) as bf16 into
//                 TMEM, row sums;
//     warps 12-15 epilogue: O / sum as bf16, stored chunk-major per pair so
//                 that the r heads of a member (consecutive lanes) write
//                 whole lines, and the log2 sum per pair;
//   pa_merge_kernel     per row and group: log-sum-exp of its pairs -> o, lse
//                       (pa_merge_many_kernel for lists beyond 32 blocks).
#include "tcgen05.cuh"

namespace msa {

namespace {

constexpr int kPtRows = 128;
constexpr int kPtSm0 = 4;       // first softmax warp
constexpr int kPtEpiWarps = 4;
constexpr int kMaxSpq = 4;      // softmax warps per TMEM lane quadrant: BK / 32 (32 keys each)
// warps of the tile kernel for a block size: 4 control warps, 4 * BK / 32 softmax warps, 4 epilogue warps
__host__ __device__ constexpr int pt_threads(int bk) { return (4 + 4 * (bk / 32) + kPtEpiWarps) * 32; }
constexpr int kHalf = 16384;    // one 128-row x 128-byte operand tile
constexpr int kInfoSlots = 6;   // tiles staged ahead in shared memory
// every role but the stager releases a tile's info slot: K/V producer, MMA issuer, Q gather,
// the softmax warps, the epilogue warps
__host__ __device__ constexpr int info_consumers(int bk) { return 3 + 4 * (bk / 32) + kPtEpiWarps; }
constexpr int kRun = 8;         // consecutive tiles of the list a CTA takes at a time

// One tile as the roles read it: its block, members, and whether the next tile changes block.
struct TileInfo {
    int bkt, start, cnt, last;  // last: the CTA's next tile is another bucket (or none)
    int b, g, n, pad;
    int mem[kPtRows];           // member i: (row tt << kSlotBits) | slot
};

struct PtBars {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2];
    uint64_t o_full[2], o_empty[2];
    uint64_t ml_full[2], ml_empty[2];
    uint64_t info_full[kInfoSlots], info_empty[kInfoSlots];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    float red_m[2][kMaxSpq][kPtRows];  // [buffer][key part][row] raw max of the part
    float ml_m[2][kPtRows];            // [buffer][row] row max, log2 domain
    float ml_l[2][kMaxSpq][kPtRows];   // [buffer][key part][row] sum of the part
    TileInfo info[kInfoSlots];
};

__device__ inline void mbar_arrive1(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x 16 bf16) read from tensor memory, lane i = row i,
// two bf16 per 32-bit column, lower k in the low half; the accumulate flag fixed at compile time.
template <bool ACC>
__device__ inline void mma_bf16_ts_c(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "n"(ACC ? 1 : 0)
        : "memory");
}

template <int N>
__device__ inline void tmem_st(uint32_t taddr, const uint32_t (&r)[N]);
template <>
__device__ inline void tmem_st<16>(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
template <>
__device__ inline void tmem_st<32>(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ inline void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x for x <= 0 on the FMA pipe, so that part of the softmax's exponentials leave the MUFU
// unit: x is clamped at -125 (2^-125 stands for anything smaller, also for -inf), rounded to the
// nearest integer n by adding 1.5 * 2^23 (n then sits in the low mantissa bits, and n << 23 equals
// those bits shifted by 23), 2^(x - n) with x - n in [-1/2, 1/2] comes from a cubic fitted to 2^f
// by least squares in relative error at Chebyshev nodes (max relative error 7.5e-5, against the
// 2^-9 of the bf16 that P is stored in), and 2^n is added to its exponent field.
__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -125.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    float p = fmaf(f, 0.0551716648f, 0.242611125f);
    p = fmaf(p, f, 0.693260968f);
    p = fmaf(p, f, 0.999928057f);
    return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// 2^x with the hardware approximation (2^-inf = +0).
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Barrier over the softmax warps of one lane quadrant (nthreads threads) that also ANDs a
// per-thread flag across them, so all of them leave a loop at the same barrier when any has
// given up a wait.
__device__ inline bool quad_sync_and(int id, int nthreads, bool ok) {
    uint32_t r;
    __syncwarp();
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle layout: 64-element
// rows of 128 bytes along N, consecutive K rows 128 bytes apart, 8-row groups 1024 bytes apart
// (stride byte offset), the next 64 elements of N `lbo` bytes further (leading byte offset).
__device__ inline uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// A pair (row t of the pass, slot j of its list, group g, sequence b) is attended when its
// block is visible to the row.
__device__ inline bool pair_valid(int id, int bk, int pos) { return id >= 0 && id * bk <= pos; }

// ------------------------------------------------------------------ bucketing
__global__ void pa_count_kernel(const PrefillAttnArgs a) {
    const long long n = (long long)a.B * a.Tn * a.G * a.k;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int j = (int)(i % a.k);
        long long rest = i / a.k;
        const int g = (int)(rest % a.G);
        rest /= a.G;
        const int tt = (int)(rest % a.Tn);
        const int b = (int)(rest / a.Tn);
        const int t = a.t0 + tt;
        const int id = a.ids[(((size_t)b * a.T + t) * a.G + g) * a.k + j];
        int rk = -1;
        if (pair_valid(id, a.Bk, a.q_start + t) && id < a.nbv)
            rk = atomicAdd(&a.counts[((size_t)b * a.G + g) * a.nbv + id], 1);
        a.rank[i] = rk;
    }
}

// Block-wide sum of (x, y) over 1024 threads; every thread gets the totals.
__device__ inline void block_sum2(long long &x, long long &y, long long (*sh)[2]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x += __shfl_xor_sync(FULL, x, o);
        y += __shfl_xor_sync(FULL, y, o);
    }
    __syncthreads();
    if (lane == 0) { sh[warp][0] = x; sh[warp][1] = y; }
    __syncthreads();
    x = lane < (int)(blockDim.x >> 5) ? sh[lane][0] : 0;
    y = lane < (int)(blockDim.x >> 5) ? sh[lane][1] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x += __shfl_xor_sync(FULL, x, o);
        y += __shfl_xor_sync(FULL, y, o);
    }
}

// Pairs and tiles of the 1024 buckets of each scan block.
__global__ void __launch_bounds__(1024) pa_tilecount_kernel(const PrefillAttnArgs a) {
    __shared__ long long sh[32][2];
    const int nb = a.B * a.G * a.nbv;
    const int s = blockIdx.x * 1024 + threadIdx.x;
    const int c = s < nb ? a.counts[s] : 0;
    long long p = c, t = (c + a.tt - 1) / a.tt;
    block_sum2(p, t, sh);
    if (threadIdx.x == 0) {
        a.block_sums[2 * blockIdx.x] = (int)p;
        a.block_sums[2 * blockIdx.x + 1] = (int)t;
    }
}

// Exclusive scan of the bucket counts (pairs and tiles): bucket offsets and the tile list in
// bucket order.  Each block adds the totals of the blocks before it.
__global__ void __launch_bounds__(1024) pa_emit_kernel(const PrefillAttnArgs a) {
    __shared__ long long sh[32][2];
    __shared__ long long wsum[32][2];
    const int nb = a.B * a.G * a.nbv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long bp = 0, bt = 0;
    for (int i = threadIdx.x; i < (int)blockIdx.x; i += 1024) {
        bp += a.block_sums[2 * i];
        bt += a.block_sums[2 * i + 1];
    }
    block_sum2(bp, bt, sh);
    const int s = blockIdx.x * 1024 + threadIdx.x;
    const int c = s < nb ? a.counts[s] : 0;
    const long long nt = (c + a.tt - 1) / a.tt;
    long long ip = c, it = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long vp = __shfl_up_sync(FULL, ip, o), vt = __shfl_up_sync(FULL, it, o);
        if (lane >= o) { ip += vp; it += vt; }
    }
    if (lane == 31) { wsum[warp][0] = ip; wsum[warp][1] = it; }
    __syncthreads();
    if (warp == 0) {
        long long xp = wsum[lane][0], xt = wsum[lane][1];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long vp = __shfl_up_sync(FULL, xp, o), vt = __shfl_up_sync(FULL, xt, o);
            if (lane >= o) { xp += vp; xt += vt; }
        }
        wsum[lane][0] = xp;
        wsum[lane][1] = xt;
    }
    __syncthreads();
    long long p0 = bp + ip - c + (warp > 0 ? wsum[warp - 1][0] : 0);
    long long t0 = bt + it - nt + (warp > 0 ? wsum[warp - 1][1] : 0);
    if (s < nb) {
        a.offsets[s] = (int)p0;
        for (int q = 0; q < nt; ++q) {
            const int m = c - q * a.tt < a.tt ? c - q * a.tt : a.tt;
            a.tiles[t0 + q] = make_int4(s, (int)p0 + q * a.tt, m, 0);
        }
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 1023) *a.n_tiles = (int)(bt + wsum[31][1]);
}

__global__ void pa_scatter_kernel(const PrefillAttnArgs a) {
    const long long n = (long long)a.B * a.Tn * a.G * a.k;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int rk = a.rank[i];
        if (rk < 0) continue;
        const int j = (int)(i % a.k);
        long long rest = i / a.k;
        const int g = (int)(rest % a.G);
        rest /= a.G;
        const int tt = (int)(rest % a.Tn);
        const int b = (int)(rest / a.Tn);
        const int id = a.ids[(((size_t)b * a.T + a.t0 + tt) * a.G + g) * a.k + j];
        a.members[a.offsets[((size_t)b * a.G + g) * a.nbv + id] + rk] = (tt << kSlotBits) | j;
    }
}

// ------------------------------------------------------------------ tiles
template <int D, int BK>
__global__ void __launch_bounds__(pt_threads(BK), 1)
    pa_tile_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const PrefillAttnArgs a) {
    constexpr int NH = D / 64;               // 64-dim halves of a row
    constexpr int KVH = BK * 128;            // bytes of one 64-dim half of a K or V block tile
    constexpr int KV_STAGE = 2 * NH * KVH;   // K halves, then V halves
    constexpr int Q_STAGE = NH * kHalf;
    constexpr int SPQ = BK / 32;             // softmax warps per lane quadrant
    constexpr int SMW = 4 * SPQ;             // softmax warps
    constexpr int EPI0 = kPtSm0 + SMW;       // first epilogue warp
    constexpr int CW = 32;                   // S columns of one softmax warp
    constexpr uint32_t O_COL = 2 * BK;       // TMEM: S/P buffers [0, 2 BK), O buffers [2 BK, 2 BK + 2 D)
    constexpr uint32_t TMEM_COLS = 512;
    static_assert(2 * BK + 2 * D <= 512, "TMEM budget");

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *smQ = base;                    // [2][NH][128 rows][128 B]
    unsigned char *smKV = smQ + 2 * Q_STAGE;      // [2][K halves | V halves]
    PtBars &S = *reinterpret_cast<PtBars *>(smKV + 2 * KV_STAGE);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kv_full[i], 1); mbar_init(&S.kv_empty[i], 1);
            mbar_init(&S.q_full[i], 1); mbar_init(&S.q_empty[i], 1);
            mbar_init(&S.s_full[i], 1); mbar_init(&S.s_empty[i], 1);
            mbar_init(&S.p_full[i], SMW);
            mbar_init(&S.o_full[i], 1); mbar_init(&S.o_empty[i], kPtEpiWarps);
            mbar_init(&S.ml_full[i], SMW); mbar_init(&S.ml_empty[i], kPtEpiWarps);
        }
        for (int i = 0; i < kInfoSlots; ++i) {
            mbar_init(&S.info_full[i], 1);
            mbar_init(&S.info_empty[i], info_consumers(BK));
        }
        mbar_init(&S.mma_done, 1);
        S.abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&qmap);
        tc::prefetch_tmap(&kmap);
        tc::prefetch_tmap(&vmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(&S.tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort_flag = &S.abort_flag;

    // This CTA's tiles: runs of kRun consecutive tiles of the list (bucket order), every gridDim.x-th
    // run, so that consecutive tiles of a CTA mostly share a block (its K/V stays) while all CTAs
    // sweep the list together (the query rows of one group at a time stay in L2).
    const int nt = *a.n_tiles;
    const int n_runs = (nt + kRun - 1) / kRun;
    const int my_runs = (int)blockIdx.x < n_runs ? (n_runs - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    int n_my = my_runs * kRun;
    if (my_runs > 0 && (int)blockIdx.x + (my_runs - 1) * (int)gridDim.x == n_runs - 1) n_my -= n_runs * kRun - nt;
    auto tile_of = [&](int il) { return ((il / kRun) * (int)gridDim.x + (int)blockIdx.x) * kRun + il % kRun; };
    const int r = a.r;
    // wait for tile il's info (whole warp; false if the CTA gives up)
    auto info_wait = [&](int il) -> bool {
        bool ok = true;
        if (lane == 0) ok = tc::wait_or_abort(&S.info_full[il % kInfoSlots], (il / kInfoSlots) & 1, abort_flag, a.status);
        return __shfl_sync(FULL, ok, 0) != 0;
    };
    auto info_release = [&](int il) {
        __syncwarp();
        if (lane == 0) mbar_arrive1(&S.info_empty[il % kInfoSlots]);
    };

    if (warp == 3) {
        // ------------------------------------------------ tile info stager
        for (int il = 0; il < n_my; ++il) {
            const int ti = tile_of(il), slot = il % kInfoSlots;
            bool ok = true;
            if (lane == 0) ok = tc::wait_or_abort(&S.info_empty[slot], ((il / kInfoSlots) & 1) ^ 1, abort_flag, a.status);
            if (!__shfl_sync(FULL, ok, 0)) break;
            const int4 tile = a.tiles[ti];
            TileInfo &I = S.info[slot];
            for (int m = lane; m < tile.z; m += 32) I.mem[m] = a.members[tile.y + m];
            if (lane == 0) {
                const int bg = tile.x / a.nbv;
                I.bkt = tile.x;
                I.start = tile.y;
                I.cnt = tile.z;
                I.last = il + 1 == n_my || a.tiles[tile_of(il + 1)].x != tile.x;
                I.n = tile.x - bg * a.nbv;
                I.b = bg / a.G;
                I.g = bg - I.b * a.G;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive1(&S.info_full[slot]);
        }
    } else if (warp == 0) {
        // ------------------------------------------------ K/V producer: one load per new bucket
        int kvi = -1, prev = -1;
        for (int il = 0; il < n_my; ++il) {
            if (!info_wait(il)) break;
            const TileInfo &I = S.info[il % kInfoSlots];
            const int bkt = I.bkt, b = I.b, g = I.g, n = I.n;
            info_release(il);
            if (bkt == prev) continue;
            prev = bkt;
            ++kvi;
            const int ks = kvi & 1;
            bool ok = true;
            if (lane == 0) ok = tc::wait_or_abort(&S.kv_empty[ks], ((kvi >> 1) & 1) ^ 1, abort_flag, a.status);
            if (!__shfl_sync(FULL, ok, 0)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&S.kv_full[ks], 2 * NH * KVH);
                const int row = a.cache.row(b, g, a.G, a.L_max, n * BK);
                unsigned char *dst = smKV + ks * KV_STAGE;
                for (int h = 0; h < NH; ++h) tc::tma_load_2d(dst + h * KVH, &kmap, h * 64, row, &S.kv_full[ks]);
                for (int h = 0; h < NH; ++h)
                    tc::tma_load_2d(dst + (NH + h) * KVH, &vmap, h * 64, row, &S.kv_full[ks]);
            }
            __syncwarp();
        }
    } else if (warp == 2) {
        // ------------------------------------------------ Q gather: the members' r heads, one box per member and half
        for (int il = 0; il < n_my; ++il) {
            const int qs = il & 1;
            if (!info_wait(il)) break;
            const TileInfo &I = S.info[il % kInfoSlots];
            const int cnt = I.cnt, b = I.b, g = I.g;
            int mem[kPtRows / 32];
#pragma unroll
            for (int q = 0; q < kPtRows / 32; ++q) mem[q] = lane + 32 * q < cnt ? I.mem[lane + 32 * q] : 0;
            info_release(il);
            bool ok = true;
            if (lane == 0) ok = tc::wait_or_abort(&S.q_empty[qs], ((il >> 1) & 1) ^ 1, abort_flag, a.status);
            if (!__shfl_sync(FULL, ok, 0)) break;
            if (lane == 0) mbar_arrive_expect_tx(&S.q_full[qs], (uint32_t)cnt * r * 128 * NH);
            __syncwarp();
#pragma unroll
            for (int q = 0; q < kPtRows / 32; ++q) {
                const int m = lane + 32 * q;
                if (m < cnt) {
                    const int qrow = ((b * a.T + a.t0 + (mem[q] >> kSlotBits)) * a.Hq) + g * r;
                    for (int h = 0; h < NH; ++h)
                        tc::tma_load_2d(smQ + qs * Q_STAGE + h * kHalf + m * r * 128, &qmap, h * 64, qrow,
                                        &S.q_full[qs]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc_qk = tc::idesc_bf16_f32(kPtRows, BK);
        const uint32_t idesc_pv = tc::idesc_bf16_f32(kPtRows, D) | (1u << 16);  // B (V) is MN-major
        int kvi = -1, prev = -1;
        int pend = -1, pend_ks = 0;
        bool pend_last = false, ok = true;
        // O = P V of tile `il` (its P overwrote its S buffer); frees the S buffer and, after a
        // bucket's last tile, the K/V stage
        // descriptor bases of the Q, K and V operands in stage 0 (the issue loops only add offsets)
        const uint64_t qd0 = tc::sw128_kmajor_desc(smem_u32(smQ)), kd0 = tc::sw128_kmajor_desc(smem_u32(smKV));
        const uint64_t vd0 = sw128_mnmajor_desc(smem_u32(smKV + NH * KVH), KVH);
        auto issue_pv = [&](int il, int ks, bool last) -> bool {
            const int ob = il & 1;
            if (!tc::wait_or_abort(&S.p_full[ob], (il >> 1) & 1, abort_flag, a.status)) return false;
            if (!tc::wait_or_abort(&S.o_empty[ob], ((il >> 1) & 1) ^ 1, abort_flag, a.status)) return false;
            tc::fence_after_sync();
            const uint64_t vd = tc::desc_add(vd0, (uint32_t)(ks * KV_STAGE));
            const uint32_t od = tmem + O_COL + ob * D, pa = tmem + ob * BK;
            mma_bf16_ts_c<false>(od, pa, vd, idesc_pv);
#pragma unroll
            for (int kk = 1; kk < BK / 16; ++kk) mma_bf16_ts_c<true>(od, pa + kk * 8, tc::desc_add(vd, kk * 2048), idesc_pv);
            tc::mma_commit(&S.o_full[ob]);
            tc::mma_commit(&S.s_empty[ob]);
            if (last) tc::mma_commit(&S.kv_empty[ks]);
            return true;
        };
        for (int il = 0; il < n_my && ok; ++il) {
            const int sb = il & 1;
            if (!info_wait(il)) break;
            const TileInfo &I = S.info[il % kInfoSlots];
            const int bkt = I.bkt;
            const bool last = I.last != 0;
            info_release(il);
            if (bkt != prev) { prev = bkt; ++kvi; }
            const int ks = kvi & 1;
            if (lane == 0) {
                if (!tc::wait_or_abort(&S.q_full[sb], (il >> 1) & 1, abort_flag, a.status) ||
                    !tc::wait_or_abort(&S.kv_full[ks], (kvi >> 1) & 1, abort_flag, a.status) ||
                    !tc::wait_or_abort(&S.s_empty[sb], ((il >> 1) & 1) ^ 1, abort_flag, a.status)) {
                    ok = false;
                } else {
                    tc::fence_after_sync();
                    const uint64_t qd = tc::desc_add(qd0, (uint32_t)(sb * Q_STAGE));
                    const uint64_t kd = tc::desc_add(kd0, (uint32_t)(ks * KV_STAGE));
                    const uint32_t sd = tmem + sb * BK;
                    tc::mma_bf16_ss_c<false>(sd, qd, kd, idesc_qk);
#pragma unroll
                    for (int kk = 1; kk < D / 16; ++kk)
                        tc::mma_bf16_ss_c<true>(sd, tc::desc_add(qd, (kk >> 2) * kHalf + (kk & 3) * 32),
                                                tc::desc_add(kd, (kk >> 2) * KVH + (kk & 3) * 32), idesc_qk);
                    tc::mma_commit(&S.q_empty[sb]);
                    tc::mma_commit(&S.s_full[sb]);
                    if (pend >= 0 && !issue_pv(pend, pend_ks, pend_last)) ok = false;
                }
            }
            ok = __shfl_sync(FULL, ok, 0) != 0;
            pend = il;
            pend_ks = ks;
            pend_last = last;
        }
        if (lane == 0) {
            if (ok && pend >= 0) issue_pv(pend, pend_ks, pend_last);
            tc::mma_commit(&S.mma_done);
            mbar_wait(&S.mma_done, 0, a.status);
        }
    } else if (warp >= kPtSm0 && warp < EPI0) {
        // ------------------------------------------------ softmax
        // Warps w, w + 4, ... share TMEM lane quadrant w % 4 (one row per lane); part hf takes the
        // block's keys [hf*CW, hf*CW + CW).  Every wait of a tile comes before the quadrant
        // barrier, whose AND makes any failure uniform over the quadrant's warps.
        const int sw = warp - kPtSm0;
        const int qd = sw & 3, hf = sw >> 2;
        const int quad_bar = 1 + qd;
        const int row = qd * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        const int m_i = row / r;
        const float c = a.scale_log2;
        bool ok = true;
        for (int il = 0; il < n_my; ++il) {
            const int sb = il & 1, par = (il >> 1) & 1;
            if (ok) ok = info_wait(il);
            int n = 0, pos = 0;
            bool valid = false;
            if (ok) {
                const TileInfo &I = S.info[il % kInfoSlots];
                n = I.n;
                valid = m_i < I.cnt;
                if (valid) pos = a.q_start + a.t0 + (I.mem[m_i] >> kSlotBits);
                info_release(il);
            }
            const bool any = __any_sync(FULL, valid);
            if (ok) ok = __all_sync(FULL, tc::wait_or_abort(&S.s_full[sb], par, abort_flag, a.status));
            if (ok) ok = __all_sync(FULL, tc::wait_or_abort(&S.ml_empty[sb], par ^ 1, abort_flag, a.status));
            uint32_t zr[CW];
            float mb = -INFINITY;
            if (ok && any) {
                tc::fence_after_sync();
#pragma unroll
                for (int cc = 0; cc < CW / 32; ++cc)
                    tc::tmem_ld32(tmem + lane_addr + sb * BK + hf * CW + cc * 32,
                                  *reinterpret_cast<uint32_t(*)[32]>(&zr[cc * 32]));
                tc::tmem_ld_wait();
                // only the block holding the row's own position needs the causal mask
                const int key0 = n * BK + hf * CW;
                if (valid && key0 + CW - 1 > pos) {
#pragma unroll
                    for (int cc = 0; cc < CW; ++cc)
                        if (key0 + cc > pos) zr[cc] = __float_as_uint(-INFINITY);
                }
                float mx[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) mx[i] = -INFINITY;
#pragma unroll
                for (int cc = 0; cc < CW; cc += 8)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        mx[i] = tc::fmax3(mx[i], __uint_as_float(zr[cc + 2 * i]), __uint_as_float(zr[cc + 2 * i + 1]));
                mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            }
            S.red_m[sb][hf][row] = mb;
            ok = quad_sync_and(quad_bar, SPQ * 32, ok);
            if (!ok) break;
            // every lane of the quadrant's warps has read its S part: P may now overwrite the S buffer
            float mr = S.red_m[sb][0][row];
#pragma unroll
            for (int j = 1; j < SPQ; ++j) mr = fmaxf(mr, S.red_m[sb][j][row]);
            const float m2 = mr * c;  // row max in the log2 domain
            float ls = 0.f;
            if (any) {
                const float off = valid ? -m2 : 0.f;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                // 32 keys at a time: 16 packed pairs go to TMEM before the next 32 are exponentiated
#pragma unroll
                for (int h2 = 0; h2 < CW / 32; ++h2) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const int e = h2 * 16 + e2;
                        // one pair in four on the FMA pipe, the rest on MUFU
                        const float x0 = fmaf(__uint_as_float(zr[2 * e]), c, off);
                        const float x1 = fmaf(__uint_as_float(zr[2 * e + 1]), c, off);
                        const float p0 = (e & 3) == 3 ? exp2_poly(x0) : exp2_approx(x0);
                        const float p1 = (e & 3) == 3 ? exp2_poly(x1) : exp2_approx(x1);
                        acc[e & 3] += p0 + p1;
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        pk[e2] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
                    tmem_st<16>(tmem + lane_addr + sb * BK + hf * (CW / 2) + h2 * 16, pk);
                }
                ls = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                tmem_st_wait();
            }
            if (hf == 0) S.ml_m[sb][row] = m2;
            S.ml_l[sb][hf][row] = ls;
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive1(&S.p_full[sb]);
                mbar_arrive1(&S.ml_full[sb]);
            }
        }
    } else if (warp >= EPI0) {
        // ------------------------------------------------ epilogue: one pair row per lane
        // A pair's r x D outputs are stored chunk-major ([D / 8 chunks][r heads][8 dims]), so the r
        // heads of a member -- r consecutive lanes -- write r * 16 contiguous bytes per store.
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        const int m_i = row / r, hh = row % r;
        for (int il = 0; il < n_my; ++il) {
            const int ob = il & 1, par = (il >> 1) & 1;
            if (!info_wait(il)) break;
            bool valid;
            int pl = 0;
            {
                const TileInfo &I = S.info[il % kInfoSlots];
                valid = m_i < I.cnt;
                if (valid) {
                    const int mem = I.mem[m_i];
                    pl = ((I.b * a.Tn + (mem >> kSlotBits)) * a.G + I.g) * a.k + (mem & ((1 << kSlotBits) - 1));  // the pair's index in this pass
                }
                info_release(il);
            }
            const bool any = __any_sync(FULL, valid);
            if (!__all_sync(FULL, tc::wait_or_abort(&S.ml_full[ob], par, abort_flag, a.status))) break;
            const float m2 = S.ml_m[ob][row];
            float l = 0.f;
#pragma unroll
            for (int j = 0; j < SPQ; ++j) l += S.ml_l[ob][j][row];
            __syncwarp();
            if (lane == 0) mbar_arrive1(&S.ml_empty[ob]);
            if (!__all_sync(FULL, tc::wait_or_abort(&S.o_full[ob], par, abort_flag, a.status))) break;
            tc::fence_after_sync();
            if (any) {
                const float inv = valid && l > 0.f ? 1.f / l : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(a.part_o + (size_t)pl * r * D) + hh;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ov[32];
                    tc::tmem_ld32(tmem + lane_addr + O_COL + ob * D + cc * 32, ov);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(ov[q * 8 + 2 * e]) * inv,
                                                                            __uint_as_float(ov[q * 8 + 2 * e + 1]) * inv);
                            pk[e] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                        if (valid)  // read once, by the merge: stream past L2
                            __stcs(dst + (cc * 4 + q) * r, make_uint4(pk[0], pk[1], pk[2], pk[3]));
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive1(&S.o_empty[ob]);
            if (valid) __stcs(a.part_lse + (size_t)pl * r + hh, l > 0.f ? m2 + log2f(l) : -INFINITY);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ merge
// One warp per (sequence, row, group): the log-sum-exp combination of the row's pairs for all r
// heads of the group.  A pair's r x D bf16 partials are one contiguous block, chunk-major (16-byte
// chunk c = dims 8 (c / r) .., head c % r), read with lane l on chunks l, l + 32, ... (PER per
// lane); the r heads' outputs of the row are contiguous too (head-major), written back per chunk.
template <int PER>
__global__ void __launch_bounds__(256, 2) pa_merge_kernel(const PrefillAttnArgs a) {
    __shared__ float s_lse[8][kMaxTopKList * 16];  // per warp: [slot][head] log2 sums
    __shared__ float s_m[8][16], s_inv[8][16];     // per warp and head: max, 1 / sum of weights
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long w = blockIdx.x * 8LL + wib;
    if (w >= (long long)a.B * a.Tn * a.G) return;  // whole warps only; no block-wide barrier below
    const int g = (int)(w % a.G);
    const long long rest = w / a.G;
    const int tt = (int)(rest % a.Tn);
    const int b = (int)(rest / a.Tn);
    const int t = a.t0 + tt;
    const int pos = a.q_start + t;
    const int r = a.r, k = a.k, D = a.D;
    const int rs = __ffs(r) - 1;  // r is a power of two (it divides 128)
    const size_t pl0 = (((size_t)b * a.Tn + tt) * a.G + g) * k;
    bool v = false;
    if (lane < k) {
        const int id = a.ids[(((size_t)b * a.T + t) * a.G + g) * k + lane];
        v = pair_valid(id, a.Bk, pos) && id < a.nbv;
    }
    const unsigned vmask = __ballot_sync(FULL, v);
    float *L = s_lse[wib];
    for (int e = lane; e < k * r; e += 32) L[e] = (vmask >> (e >> rs)) & 1u ? a.part_lse[pl0 * r + e] : -INFINITY;
    __syncwarp();
    if (lane < r) {
        float m = -INFINITY;
        for (int j = 0; j < k; ++j) m = fmaxf(m, L[j * r + lane]);
        float sum = 0.f;
        if (m > -INFINITY)
            for (int j = 0; j < k; ++j) sum += exp2_approx(L[j * r + lane] - m);
        s_m[wib][lane] = m;
        s_inv[wib][lane] = sum > 0.f ? 1.f / sum : 0.f;
        if (a.lse != nullptr)
            a.lse[((size_t)b * a.T + t) * a.Hq + g * r + lane] =
                sum > 0.f ? (m + log2f(sum)) * 0.69314718055994531f : -INFINITY;
    }
    __syncwarp();
    const int nch = r * D / 8, cph = D / 8;  // chunks per pair, per head row
    float acc[PER][8];
#pragma unroll
    for (int i = 0; i < PER; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
    constexpr int NBATCH = PER >= 8 ? 1 : PER >= 4 ? 2 : 4;  // slots in flight (registers: NBATCH * PER uint4)
    unsigned mk = vmask;
    while (mk) {
        int js[NBATCH];
#pragma unroll
        for (int q = 0; q < NBATCH; ++q) {
            js[q] = mk ? __ffs(mk) - 1 : -1;
            if (mk) mk &= mk - 1;
        }
        uint4 raw[NBATCH][PER];
#pragma unroll
        for (int q = 0; q < NBATCH; ++q)
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int c = lane + 32 * i;
                raw[q][i] = make_uint4(0u, 0u, 0u, 0u);
                if (js[q] >= 0 && c < nch)
                    raw[q][i] = __ldcs(reinterpret_cast<const uint4 *>(a.part_o + (pl0 + js[q]) * r * D) + c);
            }
#pragma unroll
        for (int q = 0; q < NBATCH; ++q) {
            if (js[q] < 0) continue;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int c = lane + 32 * i;
                if (c >= nch) continue;
                const int hh = c & (r - 1);
                const float wt = exp2_approx(L[js[q] * r + hh] - s_m[wib][hh]) * s_inv[wib][hh];
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw[q][i]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h[e]);
                    acc[i][2 * e] = fmaf(wt, f.x, acc[i][2 * e]);
                    acc[i][2 * e + 1] = fmaf(wt, f.y, acc[i][2 * e + 1]);
                }
            }
        }
    }
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + (((size_t)b * a.T + t) * a.Hq + g * r) * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        if (c >= nch) continue;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 o2 = __floats2bfloat162_rn(acc[i][2 * e], acc[i][2 * e + 1]);
            pk[e] = *reinterpret_cast<const uint32_t *>(&o2);
        }
        reinterpret_cast<uint4 *>(o)[(c & (r - 1)) * cph + (c >> rs)] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

// k > kMaxTopKList: the same merge over the row's slots in chunks of 32.  A first pass over the
// chunks' log2 sums keeps each head's running maximum and rescaled sum; the second weights the
// partials.
template <int PER>
__global__ void __launch_bounds__(256, 2) pa_merge_many_kernel(const PrefillAttnArgs a) {
    __shared__ float s_lse[8][32 * 16];        // per warp: [slot of the chunk][head] log2 sums
    __shared__ float s_m[8][16], s_inv[8][16];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long w = blockIdx.x * 8LL + wib;
    if (w >= (long long)a.B * a.Tn * a.G) return;  // whole warps only; no block-wide barrier below
    const int g = (int)(w % a.G);
    const long long rest = w / a.G;
    const int tt = (int)(rest % a.Tn);
    const int b = (int)(rest / a.Tn);
    const int t = a.t0 + tt;
    const int pos = a.q_start + t;
    const int r = a.r, k = a.k, D = a.D;
    const int rs = __ffs(r) - 1;
    const size_t pl0 = (((size_t)b * a.Tn + tt) * a.G + g) * k;
    const int *row_ids = a.ids + (((size_t)b * a.T + t) * a.G + g) * k;
    float *L = s_lse[wib];
    // slots j0 .. j0 + 31: which are attended, and their log2 sums into L
    auto load_chunk = [&](int j0) -> unsigned {
        bool v = false;
        if (j0 + lane < k) {
            const int id = row_ids[j0 + lane];
            v = pair_valid(id, a.Bk, pos) && id < a.nbv;
        }
        const unsigned vm = __ballot_sync(FULL, v);
        __syncwarp();  // the previous chunk's readers are done with L
        for (int e = lane; e < 32 * r; e += 32)
            L[e] = (vm >> (e >> rs)) & 1u ? a.part_lse[(pl0 + j0) * r + e] : -INFINITY;
        __syncwarp();
        return vm;
    };
    float m = -INFINITY, sum = 0.f;  // lane < r: head `lane`
    for (int j0 = 0; j0 < k; j0 += 32) {
        load_chunk(j0);
        if (lane < r) {
            float mc = -INFINITY;
            for (int j = 0; j < 32; ++j) mc = fmaxf(mc, L[j * r + lane]);
            const float mn = fmaxf(m, mc);
            if (mn > -INFINITY) {
                sum = m > -INFINITY ? sum * exp2_approx(m - mn) : 0.f;
                for (int j = 0; j < 32; ++j) sum += exp2_approx(L[j * r + lane] - mn);
                m = mn;
            }
        }
    }
    if (lane < r) {
        s_m[wib][lane] = m;
        s_inv[wib][lane] = sum > 0.f ? 1.f / sum : 0.f;
        if (a.lse != nullptr)
            a.lse[((size_t)b * a.T + t) * a.Hq + g * r + lane] =
                sum > 0.f ? (m + log2f(sum)) * 0.69314718055994531f : -INFINITY;
    }
    __syncwarp();
    const int nch = r * D / 8, cph = D / 8;
    float acc[PER][8];
#pragma unroll
    for (int i = 0; i < PER; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
    constexpr int NBATCH = PER >= 8 ? 1 : PER >= 4 ? 2 : 4;
    for (int j0 = 0; j0 < k; j0 += 32) {
        unsigned mk = load_chunk(j0);
        while (mk) {
            int js[NBATCH];
#pragma unroll
            for (int q = 0; q < NBATCH; ++q) {
                js[q] = mk ? __ffs(mk) - 1 : -1;
                if (mk) mk &= mk - 1;
            }
            uint4 raw[NBATCH][PER];
#pragma unroll
            for (int q = 0; q < NBATCH; ++q)
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    const int c = lane + 32 * i;
                    raw[q][i] = make_uint4(0u, 0u, 0u, 0u);
                    if (js[q] >= 0 && c < nch)
                        raw[q][i] = __ldcs(reinterpret_cast<const uint4 *>(a.part_o + (pl0 + j0 + js[q]) * r * D) + c);
                }
#pragma unroll
            for (int q = 0; q < NBATCH; ++q) {
                if (js[q] < 0) continue;
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    const int c = lane + 32 * i;
                    if (c >= nch) continue;
                    const int hh = c & (r - 1);
                    const float wt = exp2_approx(L[js[q] * r + hh] - s_m[wib][hh]) * s_inv[wib][hh];
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw[q][i]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        acc[i][2 * e] = fmaf(wt, f.x, acc[i][2 * e]);
                        acc[i][2 * e + 1] = fmaf(wt, f.y, acc[i][2 * e + 1]);
                    }
                }
            }
        }
    }
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(a.o) + (((size_t)b * a.T + t) * a.Hq + g * r) * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        if (c >= nch) continue;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 o2 = __floats2bfloat162_rn(acc[i][2 * e], acc[i][2 * e + 1]);
            pk[e] = *reinterpret_cast<const uint32_t *>(&o2);
        }
        reinterpret_cast<uint4 *>(o)[(c & (r - 1)) * cph + (c >> rs)] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

template <int D, int BK>
size_t tile_smem_bytes() {
    return 1024 + 2 * (size_t)(D / 64) * kHalf + 2 * (size_t)(2 * (D / 64) * BK * 128) + sizeof(PtBars) + 64;
}

template <int D, int BK>
cudaError_t launch_tiles(const PrefillAttnArgs &a, const CUtensorMap &qm, const CUtensorMap &km, const CUtensorMap &vm,
                         int grid, cudaStream_t s) {
    const size_t smem = tile_smem_bytes<D, BK>();
    if (smem > 232448) return cudaErrorInvalidValue;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(pa_tile_kernel<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    pa_tile_kernel<D, BK><<<grid, pt_threads(BK), smem, s>>>(qm, km, vm, a);
    return cudaGetLastError();
}

}  // namespace

PrefillAttnPlan prefill_attn_plan(const msa_params_t &p) {
    PrefillAttnPlan L{};
    const int r = p.n_q_heads / p.n_kv_heads;
    const int tt = 128 / r;
    const int per_pass = prefill_rows_per_pass(p.top_k);
    L.rows = p.q_len < per_pass ? p.q_len : per_pass;
    L.nbv_max = (p.q_start + p.q_len - 1) / p.block_size + 1;
    const size_t pairs = (size_t)p.batch * L.rows * p.n_kv_heads * p.top_k;
    const size_t buckets = (size_t)p.batch * p.n_kv_heads * L.nbv_max;
    L.max_tiles = (int)(pairs / tt + buckets + 1);
    auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t off = kStatusBytes;
    L.counts = off; off += r256(buckets * 4);
    L.offsets = off; off += r256(buckets * 4);
    L.n_tiles = off; off += 256;
    L.block_sums = off; off += r256((buckets + 1023) / 1024 * 8);
    L.rank = off; off += r256(pairs * 4);
    L.members = off; off += r256(pairs * 4);
    L.tiles = off; off += r256((size_t)L.max_tiles * 16);
    L.part_lse = off; off += r256(pairs * r * 4);
    L.part_o = off; off += r256(pairs * r * p.head_dim * 2);
    L.total = off;
    return L;
}

cudaError_t launch_prefill_attn(PrefillAttnArgs a, const void *q, const void *k_cache, const void *v_cache, int n_sm,
                                cudaStream_t s, const char **why) {
    CUtensorMap qm, km, vm;
    // q as [B * T * Hq rows, D]: a box of 64 dims x r rows holds one member's r heads
    *why = "encoding the prefill attention tensor maps failed";
    if (!encode_2d(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(q), a.D,
                   (unsigned long long)a.B * a.T * a.Hq, (unsigned long long)a.D * 2, 64, a.r,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const unsigned long long rows = a.cache.rows(a.B, a.G, a.L_max);
    if (!encode_2d(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(k_cache), a.D, rows,
                   (unsigned long long)a.D * 2, 64, a.Bk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&vm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void *>(v_cache), a.D, rows,
                   (unsigned long long)a.D * 2, 64, a.Bk, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    a.tt = 128 / a.r;
    cudaError_t e = cudaSuccess;
    const int per_pass = prefill_rows_per_pass(a.k);
    for (int t0 = 0; t0 < a.T && e == cudaSuccess; t0 += per_pass) {
        a.t0 = t0;
        a.Tn = a.T - t0 < per_pass ? a.T - t0 : per_pass;
        a.nbv = (a.q_start + t0 + a.Tn - 1) / a.Bk + 1;
        const long long pairs = (long long)a.B * a.Tn * a.G * a.k;
        const int pgrid = (int)((pairs + 255) / 256 < 4LL * n_sm ? (pairs + 255) / 256 : 4LL * n_sm);
        *why = "prefill attention bucketing";
        e = cudaMemsetAsync(a.counts, 0, (size_t)a.B * a.G * a.nbv * 4, s);
        if (e != cudaSuccess) break;
        const int sgrid = (a.B * a.G * a.nbv + 1023) / 1024;
        pa_count_kernel<<<pgrid, 256, 0, s>>>(a);
        pa_tilecount_kernel<<<sgrid, 1024, 0, s>>>(a);
        pa_emit_kernel<<<sgrid, 1024, 0, s>>>(a);
        pa_scatter_kernel<<<pgrid, 256, 0, s>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) break;
        *why = "prefill attention tile launch (shared memory or shape out of range)";
        if (a.D == 128)
            e = a.Bk == 128 ? launch_tiles<128, 128>(a, qm, km, vm, n_sm, s) : launch_tiles<128, 64>(a, qm, km, vm, n_sm, s);
        else
            e = a.Bk == 128 ? launch_tiles<64, 128>(a, qm, km, vm, n_sm, s) : launch_tiles<64, 64>(a, qm, km, vm, n_sm, s);
        if (e != cudaSuccess) break;
        *why = "prefill attention merge launch";
        const long long warps = (long long)a.B * a.Tn * a.G;
        const int mgrid = (int)((warps + 7) / 8);
        const int per = (a.r * a.D / 8 + 31) / 32;  // 16-byte chunks per lane
        if (a.k > kMaxTopKList) {
            if (per <= 1) pa_merge_many_kernel<1><<<mgrid, 256, 0, s>>>(a);
            else if (per <= 2) pa_merge_many_kernel<2><<<mgrid, 256, 0, s>>>(a);
            else if (per <= 4) pa_merge_many_kernel<4><<<mgrid, 256, 0, s>>>(a);
            else pa_merge_many_kernel<8><<<mgrid, 256, 0, s>>>(a);
        } else if (per <= 1) pa_merge_kernel<1><<<mgrid, 256, 0, s>>>(a);
        else if (per <= 2) pa_merge_kernel<2><<<mgrid, 256, 0, s>>>(a);
        else if (per <= 4) pa_merge_kernel<4><<<mgrid, 256, 0, s>>>(a);
        else pa_merge_kernel<8><<<mgrid, 256, 0, s>>>(a);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace msa
