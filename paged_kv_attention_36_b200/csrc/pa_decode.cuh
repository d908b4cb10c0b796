// pa_decode.cuh -- paged decode attention for sm_100a.
//
// Work decomposition.  The decode reads, for every (sequence b, kv head g),
// the np_b = ceil(L_b / bs) pages of that sequence.  Flatten all of them in
// (b, g, page) order into one list of W pages and give each of the
// persistent CTAs (one per SM) an equal contiguous share.  A CTA's share is
// a run of "segments": whole (b, g) page lists, plus at most a partial one
// at each end.  A whole segment is finished inside the CTA and writes bf16
// output; a partial one writes an fp32 split-KV partial (normalised output,
// max logit, exp-sum) and the last CTA to finish a piece of that (b, g)
// merges the pieces by log-sum-exp (flash-decoding), so long or skewed
// contexts are split exactly where the balance needs it and nowhere else.
//
// Inside a CTA.  Warp W (the producer) walks the CTA's share, reads block
// ids from the block table and streams each (block, kv head) K tile and V
// tile (bs*D*2 contiguous bytes each, see the cache layout in pa.h) into a
// ring of R shared-memory stages with 1-D bulk async copies (the TMA
// engine), completing on a per-stage mbarrier.  Per segment it also copies
// the G query rows of kv head g (contiguous in q) into a small descriptor
// ring.  Warps 0..W-1 (consumers) take stage i when i % W equals their
// index, so each page is read by exactly one warp and no CTA-wide barrier
// is needed per page.  Each consumer warp keeps its own online-softmax
// state (running max m, running sum l, fp32 accumulator) for all G query
// heads; at a segment end the warps combine their states through shared
// memory.  Every wait on an mbarrier is bounded in time.
//
// Per-page math (SIMT, fp32).  Lane = 8 * tg + c: the 8 lanes of token
// group tg share one K row; lane c owns 16-byte chunks c, c+8, ... of the
// row, so one 128-bit shared load per lane reads 4 whole rows per warp
// without bank conflicts.  q (pre-multiplied by scale*log2(e)) lives in
// registers as fp32 pairs; products and sums use packed fp32 FMA
// (__ffma2_rn); the dot product is finished with 3 xor-shuffles; the
// softmax runs in base 2 with exp2f.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct DecodeParams {
    const uint8_t* q;             // [B][Hq][D] bf16
    const uint8_t* k_cache;       // [NB][Hkv][bs][D] bf16
    const uint8_t* v_cache;
    const int32_t* block_tables;  // [B][M]
    const int32_t* context_lens;  // [B]
    __nv_bfloat16* out;           // [B][Hq][D]
    float qscale;                 // scale * log2(e): logits in base-2 units
    int32_t B, Hq, Hkv, NB, M;
    int32_t min_pages;            // fewest pages worth giving a CTA
    int32_t* counters;            // [B*Hkv] merge tickets, zero between calls
    float* part_o;                // [grid][2][G][D] split-KV partial outputs
    float2* part_ml;              // [grid][2][G] (max logit base 2, exp-sum)
    // test hook (DUMP): every segment's partials
    int32_t dump_capacity;
    int32_t* seg_meta;
    float* seg_o;
    float* seg_m;
    float* seg_l;
    int32_t* seg_count;
};

// One segment of a CTA's share, handed from the producer to the consumers.
struct SegDesc {
    int64_t bg_start;  // flattened index of page 0 of (b, g)
    int32_t b, g;
    int32_t j0;        // first page of the segment within sequence b
    int32_t npg;       // pages in the segment; 0 marks the end of the share
    int32_t L;         // context length of b
    int32_t k0, k1;    // CTAs holding pages of (b, g); whole iff k0 == k1
    int32_t first;     // this is the CTA's first segment
    int32_t pad[6];
};
static_assert(sizeof(SegDesc) == 64, "descriptor size");

// Equal split of W pages over `grid` CTAs: CTA k gets [start(k), start(k+1)).
struct Split {
    int64_t per, rem;
    __device__ __forceinline__ int64_t start(int64_t k) const { return k * per + (k < rem ? k : rem); }
    __device__ __forceinline__ int32_t owner(int64_t pg) const {
        const int64_t big = rem * (per + 1);
        return int32_t(pg < big ? pg / (per + 1) : rem + (pg - big) / per);
    }
};

template <int D, int G, int BS, int W, int R>
struct DecodeCfg {
    static constexpr int kRow = D * 2;              // bytes of one K or V row
    static constexpr int kTile = BS * kRow;         // one (block, kv head) tile
    static constexpr int kStage = 2 * kTile;        // K tile then V tile
    static constexpr int kSegSlots = 4;
    static constexpr int kQBytes = G * kRow;
    static constexpr int kCombFloats = G * D + ((2 * G + 3) / 4) * 4;  // one warp's state, 16-byte padded
    static constexpr int kThreads = (W + 1) * 32;

    static constexpr int kRingOff = 0;
    static constexpr int kQOff = kRingOff + R * kStage;
    static constexpr int kDescOff = kQOff + kSegSlots * kQBytes;
    static constexpr int kCombOff = kDescOff + kSegSlots * int(sizeof(SegDesc));
    static constexpr int kBarOff = kCombOff + 2 * W * kCombFloats * 4;
    static constexpr int kNumBars = 2 * R + 2 * kSegSlots + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kMiscBytes = 256;
    static constexpr int kSmemBytes = kMiscOff + kMiscBytes;
    static_assert(kQBytes % 16 == 0 && kTile % 16 == 0, "bulk copies need 16-byte sizes");
    static_assert(kBarOff % 8 == 0, "mbarrier alignment");
};

// Shared scalars.
struct Misc {
    int abort;
    int is_last;
    int dump_idx;
    int found;
    int b0;
    int pad0;
    long long pre0;
    long long red[16];  // block reductions, one slot per warp (<= 16 warps)
};
static_assert(sizeof(Misc) <= 256, "misc area");

// ---------------------------------------------------------------------------
// Per-page fp32 math of one consumer warp.
template <int D, int G, int BS>
struct SimtState {
    static constexpr int NCH = D / 64;  // 16-byte chunks per lane per row
    static constexpr int ROUNDS = BS / 4;
    static constexpr int kRow = D * 2;
    static_assert(D % 64 == 0 && BS % 4 == 0, "layout");

    float2 q2[G][NCH][4];
    float2 acc[G][NCH][4];
    float m[G];
    float l[G];

    __device__ __forceinline__ void load_q(const uint8_t* qs, int c, float qscale) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const uint4 v = lds128(qs + h * kRow + (c + 8 * i) * 16);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = bf16x2_to_float2(w[j]);
                    q2[h][i][j] = make_float2(f.x * qscale, f.y * qscale);
                }
            }
    }

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
#pragma unroll
            for (int i = 0; i < NCH; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[h][i][j] = make_float2(0.f, 0.f);
        }
    }

    // One page: K tile kt, V tile vt (shared memory), rows >= nvalid masked.
    __device__ __forceinline__ void page(const uint8_t* kt, const uint8_t* vt, int nvalid, int tg, int c) {
        float s[ROUNDS][G];
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const uint8_t* row = kt + (r * 4 + tg) * kRow + c * 16;
            float2 part[G];
#pragma unroll
            for (int h = 0; h < G; ++h) part[h] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const uint4 v = lds128(row + i * 128);
                const float2 k0 = bf16x2_to_float2(v.x), k1 = bf16x2_to_float2(v.y);
                const float2 k2 = bf16x2_to_float2(v.z), k3 = bf16x2_to_float2(v.w);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    part[h] = __ffma2_rn(q2[h][i][0], k0, part[h]);
                    part[h] = __ffma2_rn(q2[h][i][1], k1, part[h]);
                    part[h] = __ffma2_rn(q2[h][i][2], k2, part[h]);
                    part[h] = __ffma2_rn(q2[h][i][3], k3, part[h]);
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) s[r][h] = part[h].x + part[h].y;
        }
        // finish each dot product across the 8 lanes of its token group
#pragma unroll
        for (int off = 1; off < 8; off <<= 1)
#pragma unroll
            for (int r = 0; r < ROUNDS; ++r)
#pragma unroll
                for (int h = 0; h < G; ++h) s[r][h] += __shfl_xor_sync(0xffffffffu, s[r][h], off);
        // rows past the context contribute nothing (their bytes may be anything)
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const bool valid = (r * 4 + tg) < nvalid;
#pragma unroll
            for (int h = 0; h < G; ++h) s[r][h] = valid ? s[r][h] : -INFINITY;
        }
        // online softmax: page max, rescale when the running max grows
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float pm = s[0][h];
#pragma unroll
            for (int r = 1; r < ROUNDS; ++r) pm = fmaxf(pm, s[r][h]);
            pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 8));
            pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 16));
            if (pm > m[h]) {  // same decision in every lane
                const float alpha = exp2f(m[h] - pm);
                const float2 a2 = make_float2(alpha, alpha);
                m[h] = pm;
                l[h] *= alpha;
#pragma unroll
                for (int i = 0; i < NCH; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[h][i][j] = __fmul2_rn(acc[h][i][j], a2);
            }
        }
        float pr[ROUNDS][G];
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r)
#pragma unroll
            for (int h = 0; h < G; ++h) {
                pr[r][h] = exp2f(s[r][h] - m[h]);
                l[h] += pr[r][h];
            }
        // P.V over the valid rows
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            if ((r * 4 + tg) < nvalid) {
                const uint8_t* row = vt + (r * 4 + tg) * kRow + c * 16;
#pragma unroll
                for (int i = 0; i < NCH; ++i) {
                    const uint4 v = lds128(row + i * 128);
                    const float2 v0 = bf16x2_to_float2(v.x), v1 = bf16x2_to_float2(v.y);
                    const float2 v2 = bf16x2_to_float2(v.z), v3 = bf16x2_to_float2(v.w);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float2 pp = make_float2(pr[r][h], pr[r][h]);
                        acc[h][i][0] = __ffma2_rn(pp, v0, acc[h][i][0]);
                        acc[h][i][1] = __ffma2_rn(pp, v1, acc[h][i][1]);
                        acc[h][i][2] = __ffma2_rn(pp, v2, acc[h][i][2]);
                        acc[h][i][3] = __ffma2_rn(pp, v3, acc[h][i][3]);
                    }
                }
            }
        }
    }

    // Sum l and acc over the 4 token groups of the warp.
    __device__ __forceinline__ void reduce_groups() {
#pragma unroll
        for (int off = 8; off < 32; off <<= 1) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
#pragma unroll
                for (int i = 0; i < NCH; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[h][i][j].x += __shfl_xor_sync(0xffffffffu, acc[h][i][j].x, off);
                        acc[h][i][j].y += __shfl_xor_sync(0xffffffffu, acc[h][i][j].y, off);
                    }
            }
        }
    }

    // Warp state -> comb[G*D + 2G]: acc[h][d], then m[h], then l[h].
    __device__ __forceinline__ void deposit(float* comb, int lane) const {
        const int tg = lane >> 3, c = lane & 7;
        if (tg == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int i = 0; i < NCH; ++i) {
                    float4* dst = reinterpret_cast<float4*>(comb + h * D + (c + 8 * i) * 8);
                    dst[0] = make_float4(acc[h][i][0].x, acc[h][i][0].y, acc[h][i][1].x, acc[h][i][1].y);
                    dst[1] = make_float4(acc[h][i][2].x, acc[h][i][2].y, acc[h][i][3].x, acc[h][i][3].y);
                }
        }
        if (lane == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                comb[G * D + h] = m[h];
                comb[G * D + G + h] = l[h];
            }
        }
    }
};

// ---------------------------------------------------------------------------
template <int BS>
__device__ __forceinline__ int32_t clamp_len(const DecodeParams& p, int b, bool report) {
    int32_t L = __ldg(p.context_lens + b);
    const int64_t cap = int64_t(p.M) * BS;
    if (L < 0 || L > cap) {
        if (report) raise_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : int32_t(cap);
    }
    return L;
}

template <int D, int G, int BS, int W, int R, bool DUMP>
__global__ void __launch_bounds__((W + 1) * 32, 1) decode_kernel(const DecodeParams p) {
    // Stage i % R always feeds warp i % W, so a warp waiting on a stage is at
    // most one phase away from it and the parity waits are exact.
    static_assert(R % W == 0, "ring depth must be a multiple of the consumer warps");
    static_assert(W + 1 <= 16, "block reductions hold 16 warps");
    using Cfg = DecodeCfg<D, G, BS, W, R>;
    constexpr int S = Cfg::kSegSlots;
    constexpr int NT = Cfg::kThreads;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem + Cfg::kRingOff;
    uint8_t* qring = smem + Cfg::kQOff;
    SegDesc* descs = reinterpret_cast<SegDesc*>(smem + Cfg::kDescOff);
    float* combbuf = reinterpret_cast<float*>(smem + Cfg::kCombOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* empty = full + R;
    uint64_t* segfull = empty + R;
    uint64_t* segempty = segfull + S;
    uint64_t* consbar = segempty + S;
    Misc* misc = reinterpret_cast<Misc*>(smem + Cfg::kMiscOff);
    volatile int* abort = &misc->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int r = 0; r < R; ++r) {
            mbar_init(&full[r], 1);
            mbar_init(&empty[r], 1);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&segfull[s], 1);
            mbar_init(&segempty[s], W);
        }
        mbar_init(consbar, W);
        misc->abort = 0;
        misc->found = 0;
        fence_mbar_init();
    }

    // ---- pass 1: pages per kv head over all sequences; zero empty ones ----
    long long local = 0;
    for (int b = threadIdx.x; b < p.B; b += NT) {
        const int32_t L = clamp_len<BS>(p, b, blockIdx.x == 0);
        local += (L + BS - 1) / BS;
        if (L == 0 && (b % int(gridDim.x)) == int(blockIdx.x)) {
            uint4* o = reinterpret_cast<uint4*>(p.out + int64_t(b) * p.Hq * D);
            for (int i = 0; i < p.Hq * D / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
    __syncthreads();  // also publishes the barrier initialisation
    if (lane == 0) misc->red[warp] = local;
    __syncthreads();
    long long total = 0;
#pragma unroll
    for (int w = 0; w < W + 1; ++w) total += misc->red[w];
    const int64_t Wt = total * p.Hkv;  // all (b, g, page) work
    if (Wt == 0) return;
    const int64_t want = (Wt + p.min_pages - 1) / p.min_pages;
    const int64_t grid_eff = want < int64_t(gridDim.x) ? want : int64_t(gridDim.x);
    if (int64_t(blockIdx.x) >= grid_eff) return;
    const Split split{Wt / grid_eff, Wt % grid_eff};
    const int64_t p_start = split.start(blockIdx.x);
    const int64_t p_end = split.start(int64_t(blockIdx.x) + 1);
    __syncthreads();  // misc->red reads done before reuse

    // ---- pass 2: find the sequence holding p_start (chunked block scan) ----
    long long carry = 0;
    for (int base = 0; base < p.B; base += NT) {
        const int b = base + threadIdx.x;
        long long v = 0;
        if (b < p.B) v = (long long)((clamp_len<BS>(p, b, false) + BS - 1) / BS) * p.Hkv;
        long long incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += t;
        }
        if (lane == 31) misc->red[warp] = incl;
        __syncthreads();
        long long before = carry;
        for (int w = 0; w < warp; ++w) before += misc->red[w];
        long long chunk_total = 0;
        for (int w = 0; w < W + 1; ++w) chunk_total += misc->red[w];
        const long long lo = before + incl - v;
        if (v > 0 && lo <= p_start && p_start < lo + v) {
            misc->b0 = b;
            misc->pre0 = lo;
            misc->found = 1;
        }
        carry += chunk_total;
        __syncthreads();
        if (misc->found) break;
    }

    if (warp == W) {
        // ======================= producer warp =======================
        int b = misc->b0;
        int64_t pre = misc->pre0;
        int32_t Lb = clamp_len<BS>(p, b, false);
        int32_t np = (Lb + BS - 1) / BS;
        const int64_t off0 = p_start - pre;
        int g = int(off0 / np);
        int j = int(off0 - int64_t(g) * np);
        int64_t pos = p_start;
        uint32_t page_i = 0, seg_i = 0;
        constexpr int C = R < 32 ? R : 32;
        bool ok = true;
        const uint64_t pol = policy_evict_first();
        while (ok && pos < p_end) {
            const int npg = int((int64_t(np - j) < p_end - pos) ? int64_t(np - j) : p_end - pos);
            if (lane == 0) {
                const int s = seg_i % S;
                if (seg_i >= S) ok = mbar_wait(&segempty[s], ((seg_i / S) - 1) & 1, abort);
                if (ok) {
                    const int64_t bg_start = pre + int64_t(g) * np;
                    SegDesc& d = descs[s];
                    d.bg_start = bg_start;
                    d.b = b;
                    d.g = g;
                    d.j0 = j;
                    d.npg = npg;
                    d.L = Lb;
                    d.k0 = split.owner(bg_start);
                    d.k1 = split.owner(bg_start + np - 1);
                    d.first = seg_i == 0;
                    mbar_arrive_expect_tx(&segfull[s], Cfg::kQBytes);
                    bulk_g2s(qring + s * Cfg::kQBytes, p.q + (int64_t(b) * p.Hq + int64_t(g) * G) * Cfg::kRow,
                             Cfg::kQBytes, &segfull[s]);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            const int32_t* bt = p.block_tables + int64_t(b) * p.M + j;
            for (int c0 = 0; ok && c0 < npg; c0 += C) {
                const int n = (npg - c0) < C ? (npg - c0) : C;
                bool lane_ok = true;
                if (lane < n) {
                    int32_t blk = __ldg(bt + c0 + lane);
                    if (blk < 0 || blk >= p.NB) {
                        raise_error(PA_DEVERR_BLOCK_ID);
                        blk = 0;
                    }
                    const uint32_t i = page_i + c0 + lane;
                    const int slot = int(i % R);
                    const uint32_t use = i / R;
                    if (use > 0) lane_ok = mbar_wait(&empty[slot], (use - 1) & 1, abort);
                    if (lane_ok) {
                        uint8_t* st = ring + slot * Cfg::kStage;
                        const int64_t src = (int64_t(blk) * p.Hkv + g) * Cfg::kTile;
                        mbar_arrive_expect_tx(&full[slot], 2 * Cfg::kTile);
                        bulk_g2s_hint(st, p.k_cache + src, Cfg::kTile, &full[slot], pol);
                        bulk_g2s_hint(st + Cfg::kTile, p.v_cache + src, Cfg::kTile, &full[slot], pol);
                    }
                }
                ok = __all_sync(0xffffffffu, lane_ok);
            }
            page_i += npg;
            ++seg_i;
            pos += npg;
            if (pos < p_end) {  // next (b, g)
                j = 0;
                if (++g == p.Hkv) {
                    g = 0;
                    pre += int64_t(p.Hkv) * np;
                    do {
                        ++b;
                        Lb = clamp_len<BS>(p, b, false);
                        np = (Lb + BS - 1) / BS;
                    } while (np == 0);
                }
            }
        }
        if (ok && lane == 0) {  // end-of-share marker
            const int s = seg_i % S;
            if (seg_i >= S) ok = mbar_wait(&segempty[s], ((seg_i / S) - 1) & 1, abort);
            if (ok) {
                descs[s].npg = 0;
                mbar_arrive(&segfull[s]);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok && lane == 0) {
            // Error path: the consumers may be gone; let every copy this warp
            // may have started land before the CTA's shared memory is freed.
            const uint32_t last = page_i + C;
            for (uint32_t i = (last > R ? last - R : 0); i < last; ++i)
                mbar_wait(&full[i % R], (i / R) & 1, nullptr, 20000000ull);
        }
        return;
    }

    // ========================= consumer warps =========================
    SimtState<D, G, BS> st;
    const int tg = lane >> 3, c = lane & 7;
    const int ct = threadIdx.x;  // 0 .. W*32-1
    uint32_t page_base = 0, seg_i = 0, cons_phase = 0;

    auto rendezvous = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(consbar);
        const bool ok = mbar_wait(consbar, cons_phase & 1, abort);
        ++cons_phase;
        return ok;
    };

    while (true) {
        const int s = seg_i % S;
        if (!mbar_wait(&segfull[s], (seg_i / S) & 1, abort)) return;
        const SegDesc d = descs[s];
        if (d.npg == 0) break;
        st.load_q(qring + s * Cfg::kQBytes, c, p.qscale);
        __syncwarp();
        if (lane == 0) mbar_arrive(&segempty[s]);
        st.reset();

        for (int k = int((uint32_t(warp) + W - page_base % W) % W); k < d.npg; k += W) {
            const uint32_t i = page_base + k;
            const int slot = int(i % R);
            if (!mbar_wait(&full[slot], (i / R) & 1, abort)) return;
            const uint8_t* stg = ring + slot * Cfg::kStage;
            const int nv = d.L - (d.j0 + k) * BS;
            st.page(stg, stg + Cfg::kTile, nv < BS ? nv : BS, tg, c);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        page_base += d.npg;

        // ---- segment end: combine the W warp states ----
        st.reduce_groups();
        float* comb = combbuf + (seg_i & 1) * W * Cfg::kCombFloats;
        st.deposit(comb + warp * Cfg::kCombFloats, lane);
        if (!rendezvous()) return;

        const bool whole = d.k0 == d.k1;
        const int my_slot = d.first ? 0 : 1;
        if (DUMP) {
            if (ct == 0) misc->dump_idx = atomicAdd(p.seg_count, 1);
            if (!rendezvous()) return;
        }
        const int dump_idx = DUMP ? misc->dump_idx : 0;
        for (int o = ct; o < G * D; o += W * 32) {
            const int h = o / D, dd = o - h * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < W; ++w) M = fmaxf(M, comb[w * Cfg::kCombFloats + G * D + h]);
            float lsum = 0.f, a = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float* cw = comb + w * Cfg::kCombFloats;
                const float sc = exp2f(cw[G * D + h] - M);
                lsum += cw[G * D + G + h] * sc;
                a += cw[h * D + dd] * sc;
            }
            const float val = a / lsum;
            if (whole) {
                p.out[(int64_t(d.b) * p.Hq + int64_t(d.g) * G + h) * D + dd] = __float2bfloat16_rn(val);
            } else {
                const int64_t ps = int64_t(blockIdx.x) * 2 + my_slot;
                p.part_o[(ps * G + h) * D + dd] = val;
                if (dd == 0) p.part_ml[ps * G + h] = make_float2(M, lsum);
            }
            if (DUMP && dump_idx < p.dump_capacity) {
                p.seg_o[(int64_t(dump_idx) * G + h) * D + dd] = val;
                if (dd == 0) {
                    p.seg_m[int64_t(dump_idx) * G + h] = M * 0.69314718055994531f;  // base 2 -> natural
                    p.seg_l[int64_t(dump_idx) * G + h] = lsum;
                }
                if (o == 0) {
                    int32_t* mt = p.seg_meta + int64_t(dump_idx) * 4;
                    mt[0] = d.b;
                    mt[1] = d.g;
                    mt[2] = d.j0 * BS;
                    const int t1 = (d.j0 + d.npg) * BS;
                    mt[3] = t1 < d.L ? t1 : d.L;
                }
            }
        }

        if (!whole) {
            // ---- split-KV: the last CTA to finish a piece of (b, g) merges ----
            __threadfence();
            if (!rendezvous()) return;
            if (ct == 0) {
                const int t = atomicAdd(p.counters + int64_t(d.b) * p.Hkv + d.g, 1);
                misc->is_last = (t == d.k1 - d.k0);
            }
            if (!rendezvous()) return;
            if (misc->is_last) {
                __threadfence();
                for (int o = ct; o < G * D; o += W * 32) {
                    const int h = o / D, dd = o - h * D;
                    float M = -INFINITY;
                    for (int k = d.k0; k <= d.k1; ++k) {
                        const int sl = split.start(k) < d.bg_start ? 1 : 0;
                        M = fmaxf(M, __ldcg(&p.part_ml[(int64_t(k) * 2 + sl) * G + h].x));
                    }
                    float lsum = 0.f, a = 0.f;
                    for (int k = d.k0; k <= d.k1; ++k) {
                        const int64_t ps = int64_t(k) * 2 + (split.start(k) < d.bg_start ? 1 : 0);
                        const float2 ml = __ldcg(&p.part_ml[ps * G + h]);
                        const float sc = ml.y * exp2f(ml.x - M);
                        lsum += sc;
                        a += sc * __ldcg(&p.part_o[(ps * G + h) * D + dd]);
                    }
                    p.out[(int64_t(d.b) * p.Hq + int64_t(d.g) * G + h) * D + dd] = __float2bfloat16_rn(a / lsum);
                }
                if (ct == 0) p.counters[int64_t(d.b) * p.Hkv + d.g] = 0;
            }
        }
        ++seg_i;
    }
}

}  // namespace pa
