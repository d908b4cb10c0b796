// pa_decode.cuh -- paged decode attention for sm_100a.
//
// Work decomposition.  The kv heads of a sequence are taken in head groups
// of HG (HG = the largest divisor of Hkv that is <= 8).  The decode reads,
// for every (sequence b, head group hg), np_b = ceil(L_b / bs) pages; a page
// is one physical block's K and V tiles for the HG heads, which sit next to
// each other in the cache.  Lay all (b, hg) out in order on one line, each
// taking np_b + X units: its pages, then X units for the fixed cost of
// finishing a segment (X = seg_weight, measured in pages).  Each persistent
// CTA (one per SM) takes an equal contiguous share of the line, a run of
// "segments": whole (b, hg) page lists, plus at most a partial one at each
// end.  A whole segment writes bf16 output; a partial one writes fp32
// split-KV partials (normalised output, max logit, exp-sum) and the last
// CTA to finish a piece of that (b, kv head) merges the pieces by
// log-sum-exp (flash-decoding), so long or skewed contexts are split exactly
// where the balance needs it and nowhere else.  A (b, kv head) in two
// pieces takes its merge ticket first: the first piece to finish publishes
// its partial with a ready flag and the other merges it with its own
// registers, so the merge adds two memory round trips to that CTA.  More
// pieces publish first and the last merges from memory, in two levels
// beyond 16 pieces: the last piece to finish in each run of 16 merges that
// run, and the last run merges the runs, so no CTA reads more than 16.
// Every merge combines normalised partials in a fixed (leaf) order, so the
// output does not depend on the order in which pieces finish: repeated
// calls give bit-identical results.
//
// Inside a CTA.  Warp 8 (the producer) walks the share, reads one block id
// per page from the block table and copies the page into a ring of R
// shared-memory stages of 32 KB: SPL stages per page (1 at head_dim 64, 2 at
// head_dim 128 with 8 heads), each holding HS = HG / SPL heads' K tiles and
// then their V tiles, moved by two tiled TMA copies (a 4-D box over
// [tile][panel][row][column], 128-byte swizzle) that complete on the
// stage's mbarrier.  Consumer warp w < HG owns kv head hg*HG + w: it reads
// its head's tiles from stage w / HS of every page, keeps the
// online-softmax state (running max m, running sum l, fp32 accumulator) of
// its G query heads, and at a segment end writes that head's output or
// partial by itself.  A stage is free again when its HS warps have read it;
// no CTA-wide barrier is taken per page or per segment.  Every wait on an
// mbarrier is bounded in time.
//
// Staged tile layout.  A (block, kv head) tile is bs = 16 rows of D bf16,
// held as D/64 panels of 16 lines x 128 bytes (panel p holds columns
// 64p .. 64p+63) with the 128-byte swizzle: the 16-byte chunk c of line t
// sits at chunk position c ^ (t % 8).  Any 8 consecutive rows read at one
// logical chunk therefore hit 8 different bank groups, which makes both the
// SIMT row reads and the tensor-core ldmatrix reads conflict-free.
//
// Per-page math, two policies:
//   SimtMath: lane = 8*tg + c; the 8 lanes of token group tg share one K
//     row, lane c owning chunks c, c+8; packed fp32 FMA (__ffma2_rn) on
//     q pre-scaled by scale*log2(e); 3 xor-shuffles finish a dot product.
//   MmaMath: the GQA group makes each page a small dense contraction, done
//     on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32 accumulate):
//     S^T[16 tokens x 8 heads] = K_page * Q^T, then O^T[D x 8] += V^T * P^T.
//     Heads beyond G are zero padding.  P (in [0, 1]) is split into a bf16
//     high part and a bf16 remainder, both multiplied, so P.V keeps ~16
//     mantissa bits; the softmax bookkeeping stays in fp32 registers.
#pragma once

#include "pa_append.cuh"
#include "pa_device.cuh"
#include "pa_prefix.cuh"
#include "pa_split.cuh"

#ifndef PA_EVICT_FIRST
#define PA_EVICT_FIRST 1  // K/V pages are read once: first candidates for L2 eviction
#endif

#ifndef PA_STAGE_K_BYTES
#define PA_STAGE_K_BYTES 16384  // K bytes of a ring stage (as many V bytes follow)
#endif

namespace pa {

struct DecodeParams {
    CUtensorMap tmap_k;           // K cache as [rows = NB*Hkv*bs][D/64 panels][64] bf16
    CUtensorMap tmap_v;           // V cache, same
    const uint8_t* q;             // [B][Hq][D] bf16
    const int32_t* block_tables;  // [B][M]
    const int32_t* context_lens;  // [B]
    __nv_bfloat16* out;           // [B][Hq][D]
    float qscale;                 // scale * log2(e): logits in base-2 units
    int32_t B, Hq, Hkv, NB, M;
    int32_t HG, NG;               // kv heads per head group (<= 8), head groups per sequence
    int32_t HS, SPL, SPL_LOG;     // kv heads per ring stage, stages per page (HG = HS * SPL, SPL = 2^SPL_LOG)
    int32_t min_pages;            // fewest pages worth giving a CTA
    int32_t seg_weight;           // cost of finishing a segment, in pages (weights the split)
    int32_t* counters;            // [B*Hkv] merge tickets, zero between calls
    int32_t* slot_sync;           // [grid][2][HG], per partial slot: a ready flag (a (b, kv head) in two
                                  // pieces) or a run ticket (> 16 pieces); zero between calls
    float* part_o;                // [grid][2][HG*G][D] split-KV partial outputs
    float2* part_ml;              // [grid][2][HG*G] (max logit base 2, exp-sum)
    // test hook (DUMP): every segment's partials
    int32_t dump_capacity;
    int32_t* seg_meta;
    float* seg_o;
    float* seg_m;
    float* seg_l;
    int32_t* seg_count;
    // fused append (APPEND): slot-mapped rows written before any page is read
    const uint4* k_new;           // [T][Hkv][D] bf16 as 16-byte chunks
    const uint4* v_new;
    const int32_t* slot_mapping;  // [T]
    int64_t app_chunks;           // T * Hkv * D / 8
    int32_t app_tokens;           // T
    int32_t app_local;            // 1: readers write the rows of the blocks they read (T <= kLocalMaxTokens),
                                  // 0: a grid barrier (a cooperative launch)
    uint4* k_cache_w;             // the caches, writable
    uint4* v_cache_w;
    unsigned int* grid_bar;       // {arrivals, departures}: zero between calls
    // shared prefixes (num_groups > 0): group i = sequences [off[i], off[i+1]),
    // whose first group_prefix_pages[i] pages were attended by prefix_kernel
    const int32_t* group_offsets;       // [num_groups + 1]
    const int32_t* group_prefix_pages;  // [num_groups]
    int32_t num_groups, max_group_size;
    int32_t prefix_splits;              // key ranges of the prefix partials
    // CTAs 0 .. early_ctas-1 start on SMs the prefix pass leaves free and take
    // the units one CTA streams while the pass runs more than the others:
    // early_units_per_ms * (early_ns + early_ns_per_page * pages of a key range) / 1e6
    int32_t early_ctas;
    int32_t early_ns, early_ns_per_page, early_units_per_ms;
    int32_t defer_dep;                  // 1: the decode owns the step's append, so it waits for the
                                        // prefix pass (griddepcontrol.wait) only before reading its
                                        // partials; 0: before reading anything (the pass appended)
    const float* prefix_o;              // [splits][B][Hq][D]
    const float2* prefix_ml;            // [splits][B][Hq] (max logit base 2, exp-sum)
    // fp8 caches: value = e4m3 code * scale[kv head] (null for bf16 caches)
    const float* k_scale;               // [Hkv]
    const float* v_scale;               // [Hkv]
};

// One segment of a CTA's share, handed from the producer to the consumers.
struct SegDesc {
    int32_t b, hg;     // sequence, head group
    int32_t j0;        // first page of the segment within sequence b
    int32_t npg;       // pages in the segment; 0 marks the end of the share
    int32_t L;         // context length of b
    int32_t k0, k1;    // CTAs holding pages of (b, hg); whole iff k0 == k1
    int32_t P;         // shared-prefix pages of b (the line holds pages P .. ceil(L/bs)-1)
    int32_t pad[8];
};
static_assert(sizeof(SegDesc) == 64, "descriptor size");


// Shared scalars.
struct Misc {
    int abort;
    int all_dirty;       // fused append: every page counts as written this step
    int b0;              // sequence where the share starts
    int L0, P0, np0;     // its context length, shared-prefix pages and own pages
    int pmax;            // the longest shared prefix, in pages (early CTAs only)
    long long pre0;      // weighted position of b0's first unit
    long long red[16];  // block reductions, one slot per warp (<= 16 warps)
    unsigned char patch[32];  // fused append, local: per ring stage, the consumers write the new row
};
constexpr int kMaxRing = 32;  // ring stages a decode CTA may have (Misc::patch)
static_assert(sizeof(Misc) <= 256, "misc area");


// A finished partial is read from global memory (written by other CTAs or
// by the shared-prefix pass: L2, not L1) or from this warp's shared-memory
// staging.
template <bool SMEM, class T>
__device__ __forceinline__ T ld_part(const T* p) {
    if constexpr (SMEM)
        return *p;
    else
        return __ldcg(p);
}

// ===========================================================================
// SIMT math policy.
template <int D, int G, int BS>
struct SimtMath {
    static constexpr int NCH = D / 64;  // 16-byte chunks per lane per row
    static constexpr int ROUNDS = BS / 4;
    static constexpr bool kZeroMaskedV = false;  // masked rows are skipped
    static_assert(D % 64 == 0 && BS % 4 == 0, "layout");

    static constexpr int kElemBytes = 2;  // bf16 caches
    static constexpr bool kPairPages = false;
    float2 q2[G][NCH][4];
    float2 acc[G][NCH][4];
    float m[G];
    float l[G];
    float oscale = 1.f;  // output scale (1 for bf16 caches)

    // q of the G query heads of one kv head (G rows of D bf16, global
    // memory), pre-scaled by scale * log2(e).
    __device__ __forceinline__ void load_q_global(const uint8_t* gq, int lane, float qscale) {
        const int c = lane & 7;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(gq + h * D * 2 + (c + 8 * i) * 16));
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

    __device__ __forceinline__ void page(const uint8_t* kt, const uint8_t* vt, int nvalid, int lane) {
        const int tg = lane >> 3, c = lane & 7;
        float s[ROUNDS][G];
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const int t = r * 4 + tg;
            float2 part[G];
#pragma unroll
            for (int h = 0; h < G; ++h) part[h] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const uint4 v = lds128(kt + tile_off(t, c + 8 * i));
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
#pragma unroll
        for (int off = 1; off < 8; off <<= 1)
#pragma unroll
            for (int r = 0; r < ROUNDS; ++r)
#pragma unroll
                for (int h = 0; h < G; ++h) s[r][h] += __shfl_xor_sync(0xffffffffu, s[r][h], off);
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const bool valid = (r * 4 + tg) < nvalid;
#pragma unroll
            for (int h = 0; h < G; ++h) s[r][h] = valid ? s[r][h] : -INFINITY;
        }
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
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const int t = r * 4 + tg;
            if (t < nvalid) {
#pragma unroll
                for (int i = 0; i < NCH; ++i) {
                    const uint4 v = lds128(vt + tile_off(t, c + 8 * i));
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

    // A finished partial to fold into the state (SIMT: read when folded).
    struct Piece {
        const float* o;
        const float2* ml;
    };
    __device__ __forceinline__ void piece_load(Piece& pc, const float* o, const float2* ml, int) const {
        pc.o = o;
        pc.ml = ml;
    }
    __device__ __forceinline__ void piece_absorb(const Piece& pc, int lane) { absorb(pc.o, pc.ml, lane); }

    // Folds a finished partial (normalised output o[G][D], (max logit base
    // 2, exp-sum) per head) into the state, as if its tokens had been paged
    // here.  The sums live in token group 0; every lane keeps the same m.
    template <bool SMEM = false>
    __device__ __forceinline__ void absorb(const float* o, const float2* ml, int lane) {
        const int tg = lane >> 3, c = lane & 7;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float2 pml = ld_part<SMEM>(ml + h);
            const float M = fmaxf(m[h], pml.x);
            const float a_old = exp2f(m[h] - M), a_new = pml.y * exp2f(pml.x - M);
            m[h] = M;
            l[h] = l[h] * a_old + (tg == 0 ? a_new : 0.f);
#pragma unroll
            for (int i = 0; i < NCH; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 v = make_float2(0.f, 0.f);
                    if (tg == 0) v = ld_part<SMEM>(reinterpret_cast<const float2*>(o + h * D + (c + 8 * i) * 8 + 2 * j));
                    acc[h][i][j] = make_float2(acc[h][i][j].x * a_old + a_new * v.x,
                                               acc[h][i][j].y * a_old + a_new * v.y);
                }
        }
    }

    // Sum l and acc over the 4 token groups of the warp.
    __device__ __forceinline__ void finish() {
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

    // After finish(): out[h][:] = acc / l in bf16, for the G heads.
    __device__ __forceinline__ void store_out(__nv_bfloat16* out, int lane) const {
        const int tg = lane >> 3, c = lane & 7;
        if (tg != 0) return;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float inv = oscale / l[h];
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                uint4 v;
                v.x = float2_to_bf16x2(acc[h][i][0].x * inv, acc[h][i][0].y * inv);
                v.y = float2_to_bf16x2(acc[h][i][1].x * inv, acc[h][i][1].y * inv);
                v.z = float2_to_bf16x2(acc[h][i][2].x * inv, acc[h][i][2].y * inv);
                v.w = float2_to_bf16x2(acc[h][i][3].x * inv, acc[h][i][3].y * inv);
                *reinterpret_cast<uint4*>(out + h * D + (c + 8 * i) * 8) = v;
            }
        }
    }
    // After finish(): out[h][:] (bf16) = the log-sum-exp merge of this
    // state with the finished partial pc of the same (b, kv head), both
    // taken as normalised partials (this state as store_partial would write
    // it) and combined in leaf order (this one first iff mine_first): the
    // result does not depend on which of the two pieces finished last.
    __device__ __forceinline__ void store_merged2(const Piece& pc, bool mine_first, __nv_bfloat16* out,
                                                  int lane) const {
        const int tg = lane >> 3, c = lane & 7;
        if (tg != 0) return;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float2 oml = __ldcg(pc.ml + h);
            const float inv = 1.f / l[h];
            const float ma = mine_first ? m[h] : oml.x, la = mine_first ? l[h] : oml.y;
            const float mb = mine_first ? oml.x : m[h], lb = mine_first ? oml.y : l[h];
            const float M = fmaxf(ma, mb);
            const float wa = la * exp2f(ma - M), wb = lb * exp2f(mb - M);
            const float r = oscale / (wa + wb);
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const float4* src = reinterpret_cast<const float4*>(pc.o + h * D + (c + 8 * i) * 8);
                const float4 q0 = __ldcg(src), q1 = __ldcg(src + 1);
                const float other[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                float res[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float own0 = acc[h][i][j].x * inv, own1 = acc[h][i][j].y * inv;
                    const float a0 = mine_first ? own0 : other[2 * j], b0 = mine_first ? other[2 * j] : own0;
                    const float a1 = mine_first ? own1 : other[2 * j + 1], b1 = mine_first ? other[2 * j + 1] : own1;
                    res[2 * j] = (wa * a0 + wb * b0) * r;
                    res[2 * j + 1] = (wa * a1 + wb * b1) * r;
                }
                uint4 v;
                v.x = float2_to_bf16x2(res[0], res[1]);
                v.y = float2_to_bf16x2(res[2], res[3]);
                v.z = float2_to_bf16x2(res[4], res[5]);
                v.w = float2_to_bf16x2(res[6], res[7]);
                *reinterpret_cast<uint4*>(out + h * D + (c + 8 * i) * 8) = v;
            }
        }
    }
    // After finish(): o[h][:] = acc / l (fp32) and the (max logit base 2,
    // exp-sum) pair of each head: to ml[h] if ml, else m (natural log units)
    // to mo[h] and l to lo[h].
    __device__ __forceinline__ void store_partial(float* o, float2* ml, float* mo, float* lo, int lane) const {
        const int tg = lane >> 3, c = lane & 7;
        if (tg != 0) return;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float inv = 1.f / l[h];
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                float4* dst = reinterpret_cast<float4*>(o + h * D + (c + 8 * i) * 8);
                dst[0] = make_float4(acc[h][i][0].x * inv, acc[h][i][0].y * inv, acc[h][i][1].x * inv,
                                     acc[h][i][1].y * inv);
                dst[1] = make_float4(acc[h][i][2].x * inv, acc[h][i][2].y * inv, acc[h][i][3].x * inv,
                                     acc[h][i][3].y * inv);
            }
            if (c == 0) {
                if (ml) {
                    ml[h] = make_float2(m[h], l[h]);
                } else {
                    mo[h] = m[h] * 0.69314718055994531f;
                    lo[h] = l[h];
                }
            }
        }
    }
};

// ===========================================================================
// Tensor-core math policy (mma.sync m16n8k16, bf16 x bf16 -> fp32).
// Lane roles in the 16x8 accumulator tiles: row = lane/4 (+8), column pair
// 2*(lane%4) + {0, 1}.  In S^T the rows are tokens and the columns heads;
// in O^T the rows are head-dim indices and the columns heads, so a lane
// always owns heads h0 = 2*(lane%4) and h0 + 1.
template <int D, int G, int BS>
struct MmaMath {
    static_assert(BS == 16, "one m16 tile of tokens per page");
    static_assert(G <= 8, "heads of a group fill at most the n8 tile");
    static constexpr int KS = D / 16;  // k-steps of Q.K = m-tiles of O^T
    static constexpr bool kZeroMaskedV = true;  // 0 * NaN would poison the mma

    static constexpr int kElemBytes = 2;  // bf16 caches
    static constexpr bool kPairPages = false;
    uint32_t qb[KS][2];  // Q^T as B fragments (bf16 pairs)
    float acc[KS][4];    // O^T accumulator tiles
    float m[2], l[2];    // heads h0, h0 + 1 of this lane (l: this lane's rows only)
    float qscale;
    float oscale = 1.f;  // output scale (1 for bf16 caches)

    // q of the G query heads of one kv head (G rows of D bf16, global
    // memory) as B fragments; the logits are scaled by scale * log2(e) later.
    __device__ __forceinline__ void load_q_global(const uint8_t* gq, int lane, float qs_scale) {
        qscale = qs_scale;
        const int h = lane >> 2, kk = (lane & 3) * 2;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (h < G) {
                const uint32_t* row = reinterpret_cast<const uint32_t*>(gq + h * D * 2);
                qb[ks][0] = __ldg(row + (16 * ks + kk) / 2);
                qb[ks][1] = __ldg(row + (16 * ks + kk + 8) / 2);
            } else {
                qb[ks][0] = qb[ks][1] = 0u;
            }
        }
    }

    __device__ __forceinline__ void reset() {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
#pragma unroll
        for (int i = 0; i < KS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    }

    __device__ __forceinline__ void page(const uint8_t* kt, const uint8_t* vt, int nvalid, int lane) {
        const int mi = lane >> 3, r8 = lane & 7;
        // ---- S^T = K . Q^T ----
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int t = r8 + ((mi & 1) << 3);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t a[4];
                ldmatrix_x4(a, kt + tile_off(t, 2 * ks + (mi >> 1)));
                mma_bf16_16816(s, a, qb[ks][0], qb[ks][1]);
            }
        }
        const int t0 = lane >> 2;
        const bool v0 = t0 < nvalid, v1 = (t0 + 8) < nvalid;
        s[0] = v0 ? s[0] * qscale : -INFINITY;
        s[1] = v0 ? s[1] * qscale : -INFINITY;
        s[2] = v1 ? s[2] * qscale : -INFINITY;
        s[3] = v1 ? s[3] * qscale : -INFINITY;
        // ---- online softmax over the 16 tokens of each head column ----
        float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const bool grow0 = mx0 > m[0], grow1 = mx1 > m[1];
        if (__any_sync(0xffffffffu, grow0 || grow1)) {
            const float n0 = fmaxf(m[0], mx0), n1 = fmaxf(m[1], mx1);
            const float a0 = exp2f(m[0] - n0), a1 = exp2f(m[1] - n1);
            m[0] = n0;
            m[1] = n1;
            l[0] *= a0;
            l[1] *= a1;
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                acc[i][0] *= a0;
                acc[i][1] *= a1;
                acc[i][2] *= a0;
                acc[i][3] *= a1;
            }
        }
        const float p0 = exp2f(s[0] - m[0]), p1 = exp2f(s[1] - m[1]);
        const float p2 = exp2f(s[2] - m[0]), p3 = exp2f(s[3] - m[1]);
        l[0] += p0 + p2;
        l[1] += p1 + p3;
        // ---- P^T as B fragments: bf16 high part and remainder ----
        const uint32_t h01 = float2_to_bf16x2(p0, p1), h23 = float2_to_bf16x2(p2, p3);
        const float2 f01 = bf16x2_to_float2(h01), f23 = bf16x2_to_float2(h23);
        const uint32_t r01 = float2_to_bf16x2(p0 - f01.x, p1 - f01.y);
        const uint32_t r23 = float2_to_bf16x2(p2 - f23.x, p3 - f23.y);
        const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
        const uint32_t bl0 = movmatrix_trans(r01), bl1 = movmatrix_trans(r23);
        // ---- O^T += V^T . P^T ----
        const int tv = r8 + ((mi >> 1) << 3);
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
            uint32_t a[4];
            ldmatrix_x4_trans(a, vt + tile_off(tv, 2 * mt + (mi & 1)));
            mma_bf16_16816(acc[mt], a, bh0, bh1);
            mma_bf16_16816(acc[mt], a, bl0, bl1);
        }
    }

    // A finished partial (normalised output o[G][D], (max logit base 2,
    // exp-sum) per head) held in this lane's accumulator layout, so that it
    // can be loaded when a segment starts and folded in after its pages.
    struct Piece {
        float o[KS][4];
        float2 ml[2];
    };
    template <bool SMEM = false>
    __device__ __forceinline__ void piece_load(Piece& pc, const float* o, const float2* ml, int lane) const {
        const int h0 = (lane & 3) * 2, d0 = lane >> 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = h0 + e < G ? h0 + e : 0;  // heads past G: loaded, never folded
            pc.ml[e] = ld_part<SMEM>(ml + h);
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                pc.o[mt][e] = ld_part<SMEM>(o + h * D + 16 * mt + d0);
                pc.o[mt][2 + e] = ld_part<SMEM>(o + h * D + 16 * mt + d0 + 8);
            }
        }
    }
    // Folds the piece into the state, as if its tokens had been paged here;
    // l lives in row group 0 (finish() sums the row groups).
    __device__ __forceinline__ void piece_absorb(const Piece& pc, int lane) {
        const int h0 = (lane & 3) * 2, d0 = lane >> 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (h0 + e >= G) continue;
            const float M = fmaxf(m[e], pc.ml[e].x);
            const float a_old = exp2f(m[e] - M), a_new = pc.ml[e].y * exp2f(pc.ml[e].x - M);
            m[e] = M;
            l[e] = l[e] * a_old + (d0 == 0 ? a_new : 0.f);
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                acc[mt][e] = acc[mt][e] * a_old + a_new * pc.o[mt][e];
                acc[mt][2 + e] = acc[mt][2 + e] * a_old + a_new * pc.o[mt][2 + e];
            }
        }
    }
    template <bool SMEM = false>
    __device__ __forceinline__ void absorb(const float* o, const float2* ml, int lane) {
        Piece pc;
        piece_load<SMEM>(pc, o, ml, lane);
        piece_absorb(pc, lane);
    }

    // Sum l over the 8 row groups (lanes with equal lane % 4).
    __device__ __forceinline__ void finish() {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
            l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
        }
    }

    // After finish(): out[h][:] = acc / l in bf16, for the G heads.
    __device__ __forceinline__ void store_out(__nv_bfloat16* out, int lane) const {
        const int h0 = (lane & 3) * 2, d0 = lane >> 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = h0 + e;
            if (h >= G) continue;
            const float inv = oscale / l[e];
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                out[h * D + 16 * mt + d0] = __float2bfloat16_rn(acc[mt][e] * inv);
                out[h * D + 16 * mt + d0 + 8] = __float2bfloat16_rn(acc[mt][2 + e] * inv);
            }
        }
    }
    // After finish(): out[h][:] (bf16) = the log-sum-exp merge of this
    // state with the finished partial pc of the same (b, kv head), both
    // taken as normalised partials (this state as store_partial would write
    // it) and combined in leaf order (this one first iff mine_first): the
    // result does not depend on which of the two pieces finished last.
    __device__ __forceinline__ void store_merged2(const Piece& pc, bool mine_first, __nv_bfloat16* out,
                                                  int lane) const {
        const int h0 = (lane & 3) * 2, d0 = lane >> 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = h0 + e;
            if (h >= G) continue;
            const float inv = 1.f / l[e];
            const float ma = mine_first ? m[e] : pc.ml[e].x, la = mine_first ? l[e] : pc.ml[e].y;
            const float mb = mine_first ? pc.ml[e].x : m[e], lb = mine_first ? pc.ml[e].y : l[e];
            const float M = fmaxf(ma, mb);
            const float wa = la * exp2f(ma - M), wb = lb * exp2f(mb - M);
            const float r = oscale / (wa + wb);
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float own = acc[mt][2 * k + e] * inv, other = pc.o[mt][2 * k + e];
                    const float a = mine_first ? own : other, b = mine_first ? other : own;
                    out[h * D + 16 * mt + d0 + 8 * k] = __float2bfloat16_rn((wa * a + wb * b) * r);
                }
            }
        }
    }
    // After finish(): o[h][:] = acc / l (fp32) and the (max logit base 2,
    // exp-sum) pair of each head: to ml[h] if ml, else m (natural log units)
    // to mo[h] and l to lo[h].
    __device__ __forceinline__ void store_partial(float* o, float2* ml, float* mo, float* lo, int lane) const {
        const int h0 = (lane & 3) * 2, d0 = lane >> 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = h0 + e;
            if (h >= G) continue;
            const float inv = 1.f / l[e];
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                o[h * D + 16 * mt + d0] = acc[mt][e] * inv;
                o[h * D + 16 * mt + d0 + 8] = acc[mt][2 + e] * inv;
            }
            if (d0 == 0) {
                if (ml) {
                    ml[h] = make_float2(m[e], l[e]);
                } else {
                    mo[h] = m[e] * 0.69314718055994531f;
                    lo[h] = l[e];
                }
            }
        }
    }
};

// ===========================================================================
// fp8 (E4M3) caches on the tensor cores.  K tiles arrive as [16 tokens][D]
// codes in 128-byte lines (128-byte swizzle; at head_dim 64 a line holds two
// tokens), V tiles transposed as [D][16] codes in 16-byte rows with the
// token order of pa_append.cuh.  A plain ldmatrix of 8 rows x 16 bytes gives
// each lane 4 consecutive codes of one row; each half converts exactly to an
// f16x2.  With Q^T's d order permuted the same way (k slots 2c, 2c+1 <- d
// 4c, 4c+1 and 2c+8, 2c+9 <- d 4c+2, 4c+3 within each 16) the K fragments
// feed mma.sync m16n8k16 (f16 in, fp32 accumulate); for V^T the stored
// token order makes the same conversion give tokens 2c, 2c+1, 2c+8, 2c+9,
// the natural fragment order, so P^T is the bf16 policy's, in f16.  Tokens
// past the context are zeroed in the V^T fragments (0 * NaN would poison
// the sum).  The kv head's K scale is folded into qscale and its V scale
// into oscale; the state, merges and outputs are MmaMath's.
template <int D, int G, int BS>
struct Fp8MmaMath : MmaMath<D, G, BS> {
    using Base = MmaMath<D, G, BS>;
    using Base::KS;
    using Base::qb;
    using Base::acc;
    using Base::m;
    using Base::l;
    using Base::qscale;
    static constexpr bool kZeroMaskedV = false;  // masked in the fragments
    static constexpr int kElemBytes = 1;
    static constexpr bool kPairPages = true;     // page2(): two pages per softmax update
    static_assert(D == 64 || D == 128, "128-byte K lines hold one or two tokens");

    __device__ __forceinline__ void load_q_global(const uint8_t* gq, int lane, float qs_scale) {
        qscale = qs_scale;
        const int h = lane >> 2, c = lane & 3;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (h < G) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(gq + (h * D + 16 * ks + 4 * c) * 2));
                const float2 a = bf16x2_to_float2(w.x), b = bf16x2_to_float2(w.y);
                qb[ks][0] = float2_to_f16x2(a.x, a.y);
                qb[ks][1] = float2_to_f16x2(b.x, b.y);
            } else {
                qb[ks][0] = qb[ks][1] = 0u;
            }
        }
    }

    // Byte offset of 16-byte chunk ch (d 16ch .. 16ch+15) of token t in a K tile.
    static __device__ __forceinline__ int k_off(int t, int ch) {
        const int line = D == 128 ? t : (t >> 1);
        const int lch = D == 128 ? ch : (((t & 1) << 2) + ch);
        return (line << 7) + ((lch ^ (line & 7)) << 4);
    }
    static __device__ __forceinline__ uint32_t lo(uint32_t r) { return e4m3x2_to_f16x2(uint16_t(r & 0xffffu)); }
    static __device__ __forceinline__ uint32_t hi(uint32_t r) { return e4m3x2_to_f16x2(uint16_t(r >> 16)); }

    __device__ __forceinline__ void page(const uint8_t* kt, const uint8_t* vt, int nvalid, int lane) {
        const int mi = lane >> 3, r8 = lane & 7, c = lane & 3;
        // ---- S^T = K . Q^T, two k-steps per ldmatrix ----
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int t = r8 + ((mi & 1) << 3);
#pragma unroll
            for (int j = 0; j < KS / 2; ++j) {
                uint32_t r[4];
                ldmatrix_x4(r, kt + k_off(t, 2 * j + (mi >> 1)));
                const uint32_t a0[4] = {lo(r[0]), lo(r[1]), hi(r[0]), hi(r[1])};
                mma_f16_16816(s, a0, qb[2 * j][0], qb[2 * j][1]);
                const uint32_t a1[4] = {lo(r[2]), lo(r[3]), hi(r[2]), hi(r[3])};
                mma_f16_16816(s, a1, qb[2 * j + 1][0], qb[2 * j + 1][1]);
            }
        }
        const int t0 = lane >> 2;
        const bool v0 = t0 < nvalid, v1 = (t0 + 8) < nvalid;
        s[0] = v0 ? s[0] * qscale : -INFINITY;
        s[1] = v0 ? s[1] * qscale : -INFINITY;
        s[2] = v1 ? s[2] * qscale : -INFINITY;
        s[3] = v1 ? s[3] * qscale : -INFINITY;
        // ---- online softmax over the 16 tokens of each head column ----
        float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        if (__any_sync(0xffffffffu, mx0 > m[0] || mx1 > m[1])) {
            const float n0 = fmaxf(m[0], mx0), n1 = fmaxf(m[1], mx1);
            const float a0 = exp2f(m[0] - n0), a1 = exp2f(m[1] - n1);
            m[0] = n0;
            m[1] = n1;
            l[0] *= a0;
            l[1] *= a1;
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                acc[i][0] *= a0;
                acc[i][1] *= a1;
                acc[i][2] *= a0;
                acc[i][3] *= a1;
            }
        }
        const float p0 = exp2f(s[0] - m[0]), p1 = exp2f(s[1] - m[1]);
        const float p2 = exp2f(s[2] - m[0]), p3 = exp2f(s[3] - m[1]);
        l[0] += p0 + p2;
        l[1] += p1 + p3;
        // ---- P^T as f16 B fragments ----
        const uint32_t b0 = movmatrix_trans(float2_to_f16x2(p0, p1));
        const uint32_t b1 = movmatrix_trans(float2_to_f16x2(p2, p3));
        // ---- O^T += V^T . P^T, two m-tiles (32 rows of V^T) per ldmatrix;
        // this lane's tokens: 2c, 2c+1 (low halves) and 2c+8, 2c+9 (high) ----
        const uint32_t mlo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t mhi = (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
        for (int j = 0; j < KS / 2; ++j) {
            uint32_t r[4];
            ldmatrix_x4(r, vt + (32 * j + lane) * 16);
            const uint32_t a0[4] = {lo(r[0]) & mlo, lo(r[1]) & mlo, hi(r[0]) & mhi, hi(r[1]) & mhi};
            mma_f16_16816(acc[2 * j], a0, b0, b1);
            const uint32_t a1[4] = {lo(r[2]) & mlo, lo(r[3]) & mlo, hi(r[2]) & mhi, hi(r[3]) & mhi};
            mma_f16_16816(acc[2 * j + 1], a1, b0, b1);
        }
    }

    // Two pages at once (nv1 == 0: the second is absent): both S products in
    // flight together, one max / rescale over the 32 tokens, then both P.V.
    __device__ __forceinline__ void page2(const uint8_t* kt0, const uint8_t* vt0, int nv0, const uint8_t* kt1,
                                          const uint8_t* vt1, int nv1, int lane) {
        const int mi = lane >> 3, r8 = lane & 7, c = lane & 3;
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int t = r8 + ((mi & 1) << 3);
#pragma unroll
            for (int j = 0; j < KS / 2; ++j) {
                uint32_t r[4], u[4];
                ldmatrix_x4(r, kt0 + k_off(t, 2 * j + (mi >> 1)));
                ldmatrix_x4(u, kt1 + k_off(t, 2 * j + (mi >> 1)));
                const uint32_t a0[4] = {lo(r[0]), lo(r[1]), hi(r[0]), hi(r[1])};
                const uint32_t c0[4] = {lo(u[0]), lo(u[1]), hi(u[0]), hi(u[1])};
                mma_f16_16816(s0, a0, qb[2 * j][0], qb[2 * j][1]);
                mma_f16_16816(s1, c0, qb[2 * j][0], qb[2 * j][1]);
                const uint32_t a1[4] = {lo(r[2]), lo(r[3]), hi(r[2]), hi(r[3])};
                const uint32_t c1[4] = {lo(u[2]), lo(u[3]), hi(u[2]), hi(u[3])};
                mma_f16_16816(s0, a1, qb[2 * j + 1][0], qb[2 * j + 1][1]);
                mma_f16_16816(s1, c1, qb[2 * j + 1][0], qb[2 * j + 1][1]);
            }
        }
        const int t0 = lane >> 2;
        const bool v00 = t0 < nv0, v01 = (t0 + 8) < nv0, v10 = t0 < nv1, v11 = (t0 + 8) < nv1;
        s0[0] = v00 ? s0[0] * qscale : -INFINITY;
        s0[1] = v00 ? s0[1] * qscale : -INFINITY;
        s0[2] = v01 ? s0[2] * qscale : -INFINITY;
        s0[3] = v01 ? s0[3] * qscale : -INFINITY;
        s1[0] = v10 ? s1[0] * qscale : -INFINITY;
        s1[1] = v10 ? s1[1] * qscale : -INFINITY;
        s1[2] = v11 ? s1[2] * qscale : -INFINITY;
        s1[3] = v11 ? s1[3] * qscale : -INFINITY;
        // ---- one online-softmax step over the 32 tokens of each head column ----
        float mx0 = fmaxf(fmaxf(s0[0], s0[2]), fmaxf(s1[0], s1[2]));
        float mx1 = fmaxf(fmaxf(s0[1], s0[3]), fmaxf(s1[1], s1[3]));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        if (__any_sync(0xffffffffu, mx0 > m[0] || mx1 > m[1])) {
            const float n0 = fmaxf(m[0], mx0), n1 = fmaxf(m[1], mx1);
            const float a0 = exp2f(m[0] - n0), a1 = exp2f(m[1] - n1);
            m[0] = n0;
            m[1] = n1;
            l[0] *= a0;
            l[1] *= a1;
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                acc[i][0] *= a0;
                acc[i][1] *= a1;
                acc[i][2] *= a0;
                acc[i][3] *= a1;
            }
        }
        const float p00 = exp2f(s0[0] - m[0]), p01 = exp2f(s0[1] - m[1]);
        const float p02 = exp2f(s0[2] - m[0]), p03 = exp2f(s0[3] - m[1]);
        const float p10 = exp2f(s1[0] - m[0]), p11 = exp2f(s1[1] - m[1]);
        const float p12 = exp2f(s1[2] - m[0]), p13 = exp2f(s1[3] - m[1]);
        l[0] += (p00 + p02) + (p10 + p12);
        l[1] += (p01 + p03) + (p11 + p13);
        const uint32_t b00 = movmatrix_trans(float2_to_f16x2(p00, p01));
        const uint32_t b01 = movmatrix_trans(float2_to_f16x2(p02, p03));
        const uint32_t b10 = movmatrix_trans(float2_to_f16x2(p10, p11));
        const uint32_t b11 = movmatrix_trans(float2_to_f16x2(p12, p13));
        uint32_t ml0 = 0xffffffffu, mh0 = 0xffffffffu, ml1 = 0xffffffffu, mh1 = 0xffffffffu;
        if (nv0 < 16) {
            ml0 = (2 * c < nv0 ? 0x0000ffffu : 0u) | (2 * c + 1 < nv0 ? 0xffff0000u : 0u);
            mh0 = (2 * c + 8 < nv0 ? 0x0000ffffu : 0u) | (2 * c + 9 < nv0 ? 0xffff0000u : 0u);
        }
        if (nv1 < 16) {
            ml1 = (2 * c < nv1 ? 0x0000ffffu : 0u) | (2 * c + 1 < nv1 ? 0xffff0000u : 0u);
            mh1 = (2 * c + 8 < nv1 ? 0x0000ffffu : 0u) | (2 * c + 9 < nv1 ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int j = 0; j < KS / 2; ++j) {
            uint32_t r[4], u[4];
            ldmatrix_x4(r, vt0 + (32 * j + lane) * 16);
            ldmatrix_x4(u, vt1 + (32 * j + lane) * 16);
            const uint32_t a0[4] = {lo(r[0]) & ml0, lo(r[1]) & ml0, hi(r[0]) & mh0, hi(r[1]) & mh0};
            mma_f16_16816(acc[2 * j], a0, b00, b01);
            const uint32_t a1[4] = {lo(r[2]) & ml0, lo(r[3]) & ml0, hi(r[2]) & mh0, hi(r[3]) & mh0};
            mma_f16_16816(acc[2 * j + 1], a1, b00, b01);
            const uint32_t c0[4] = {lo(u[0]) & ml1, lo(u[1]) & ml1, hi(u[0]) & mh1, hi(u[1]) & mh1};
            mma_f16_16816(acc[2 * j], c0, b10, b11);
            const uint32_t c1[4] = {lo(u[2]) & ml1, lo(u[3]) & ml1, hi(u[2]) & mh1, hi(u[3]) & mh1};
            mma_f16_16816(acc[2 * j + 1], c1, b10, b11);
        }
    }
};

// ===========================================================================
// Consumer warps of a decode CTA: warp w < HG owns kv head hg*HG + w.
constexpr int kDecodeWarps = 8;

template <int D, int BS, int R, int EB = 2>
struct DecodeCfg {
    static constexpr int NW = kDecodeWarps;
    static constexpr int kRow = D * EB;             // bytes of one K or V row (EB bytes per value)
    static constexpr int kTile = BS * kRow;         // one (block, kv head) tile
    static constexpr int kPanel = BS * 128;         // one 64-column panel of a tile
    // K tiles of up to kHeadsPerStage heads of one block: PA_STAGE_K_BYTES, or
    // less when all NW heads' tiles are smaller (fp8 at head_dim 64)
    static constexpr int kStageK = PA_STAGE_K_BYTES < NW * kTile ? PA_STAGE_K_BYTES : NW * kTile;
    static constexpr int kStage = 2 * kStageK;        // then their V tiles
    static constexpr int kHeadsPerStage = kStageK / kTile;
    static constexpr int kMaxSpl = NW / kHeadsPerStage > 1 ? NW / kHeadsPerStage : 1;  // stages per page, at most
    static_assert(kHeadsPerStage >= 1, "a stage holds at least one head's tiles");
    static constexpr int kSegSlots = 4;
    static constexpr int kThreads = (NW + 1) * 32;

    // offsets from the 1024-byte aligned base
    static constexpr int kRingOff = 0;
    static constexpr int kDescOff = kRingOff + R * kStage;
    static constexpr int kBarOff = kDescOff + kSegSlots * int(sizeof(SegDesc));
    static constexpr int kNumBars = 2 * R + 2 * kSegSlots;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kMiscBytes = 256;
    // The rest of shared memory (at least 1 KB) is one area: the fused
    // append's bitmap of the blocks it writes (hashed by block id; kDirtyBytes,
    // or the first half of it in a shared-prefix decode) and, in a
    // shared-prefix decode, from byte kDirtyBytes / 2 on, per-warp staging of
    // the prefix range partials.
    static constexpr int kDirtyOff = kMiscOff + kMiscBytes;
    static constexpr int kDirtyBytes = 1024;
    static constexpr int kBaseBytes = kDirtyOff + kDirtyBytes + 1024;  // with the smallest area; + alignment slack
    static constexpr int kAreaBytes = ((232448 - kDirtyOff - 1024) / (NW * 16)) * (NW * 16);
    static constexpr int kSmemBytes = kDirtyOff + kAreaBytes + 1024;
    static_assert(kAreaBytes >= kDirtyBytes, "the area holds the bitmap");
    static_assert(kTile % 1024 == 0 && kStage % 1024 == 0, "TMA tile alignment (128-byte swizzle)");
    static_assert(kBarOff % 8 == 0, "mbarrier alignment");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Inclusive prefix sum of v over the NT threads of the CTA; the chunk total
// goes to `total`.  red holds one slot per warp.
template <int NT>
__device__ __forceinline__ long long block_incl_scan(long long v, long long* red, long long& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    long long before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        if (w < warp) before += red[w];
        tot += red[w];
    }
    __syncthreads();
    total = tot;
    return before + incl;
}

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

// Sequence b's context: L tokens, of which the first P pages come from its
// group's shared prefix (attended by prefix_kernel; 0 without groups) and
// np = ceil(L / bs) - P pages are streamed here.  A member whose context
// does not cover the prefix, or past max_group_size in its group, keeps all
// its pages (prefix_kernel reports it).
struct SeqPages {
    int32_t L, P, np;
};

constexpr int kFewGroups = 4;  // group tables read whole, in one round of loads

template <int BS>
__device__ __forceinline__ SeqPages seq_pages(const DecodeParams& p, int b, bool report) {
    SeqPages s;
    s.L = clamp_len<BS>(p, b, report);
    s.P = 0;
    if (p.num_groups > 0) {
        // group i holds b when off[i] <= b < off[i+1]
        const int32_t* off = p.group_offsets;
        const int ng = p.num_groups;
        int32_t P = 0, beg = 0;
        if (ng <= kFewGroups) {
            int32_t o[kFewGroups + 1], pp[kFewGroups];
#pragma unroll
            for (int i = 0; i <= kFewGroups; ++i) o[i] = i <= ng ? __ldg(off + i) : 0;
#pragma unroll
            for (int i = 0; i < kFewGroups; ++i) pp[i] = i < ng ? __ldg(p.group_prefix_pages + i) : 0;
#pragma unroll
            for (int i = 0; i < kFewGroups; ++i)
                if (i < ng && o[i] <= b && b < o[i + 1]) {
                    P = pp[i];
                    beg = o[i];
                }
        } else if (b >= __ldg(off) && b < __ldg(off + ng)) {
            int lo = 0, hi = ng;  // off[lo] <= b < off[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(off + mid) <= b) lo = mid;
                else hi = mid;
            }
            P = __ldg(p.group_prefix_pages + lo);
            beg = __ldg(off + lo);
        }
        if (P > 0 && int64_t(P) * BS <= s.L && b - beg < p.max_group_size) s.P = P;
    }
    s.np = (s.L + BS - 1) / BS - s.P;
    return s;
}

// Split-KV merge.  Pieces of a (b, kv head) are merged in registers by the
// last one when there are at most kFastMergePieces, else from memory in
// runs of at most kMergeFanIn; with at most 1024 CTAs there are at most 64 runs.
constexpr int kFastMergePieces = 2;  // one other piece in registers: fits the 168-register budget
constexpr int kMergeFanIn = 16;

// Slot index of piece `leaf` of a (b, hg) whose first piece is in CTA k0:
// leaf 0 sits in slot 1 of CTA k0, every other leaf in slot 0 of its CTA.
__device__ __forceinline__ int64_t leaf_slot(int k0, int leaf) {
    return int64_t(k0 + leaf) * 2 + (leaf == 0 ? 1 : 0);
}

// Adds this warp's arrival to a ticket counter; true in every lane of the
// warp whose arrival completes `count` (the caller has fenced its writes).
__device__ __forceinline__ bool ticket(int32_t* counter, int count, int lane) {
    int last = 0;
    if (lane == 0) last = atomicAdd(counter, 1) == count - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) __threadfence();
    return last != 0;
}

// Merges, by log-sum-exp, the split-KV partials of one warp's (b, kv head)
// held by the pieces ("leaves") off, off + stride, ... (n <= 64 of them) of
// the CTAs k0 + leaf: into out (bf16, [G][D]) if given, else into the
// partial slot of leaf `off`.  Leaf 0 sits in slot 1 of CTA k0, every other
// leaf in slot 0 of its CTA.  Lane l loads the (max, sum) of pieces l and
// l + 32 for each head; the weighted sums keep a pass's loads in flight.
constexpr int kMergeMaxPieces = 64;

template <int D, int G>
__device__ __noinline__ void merge_pieces(const DecodeParams& p, int k0, int off, int stride, int n, int HG,
                                          int warp, int lane, __nv_bfloat16* out, float oscale = 1.f) {
    auto base = [&](int i) -> int64_t {
        const int leaf = off + i * stride;
        return ((int64_t(k0 + leaf) * 2 + (leaf == 0 ? 1 : 0)) * HG + warp) * G;
    };
    float M[G], lsum[G], w[G][2];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float2 ml[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = lane + 32 * r;
            ml[r] = i < n ? __ldcg(&p.part_ml[base(i) + h]) : make_float2(-INFINITY, 0.f);
        }
        float mx = fmaxf(ml[0].x, ml[1].x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sm = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            w[h][r] = lane + 32 * r < n ? ml[r].y * exp2f(ml[r].x - mx) : 0.f;
            sm += w[h][r];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        M[h] = mx;
        lsum[h] = sm;
    }
    // pass t covers elements 128t .. 128t+127 of [G][D]: heads hl and hl + 1
    // (head_dim 64) or hl alone (head_dim 128); this lane's 4 are e .. e+3.
    // The piece loop is outermost so that every pass's load of 4 pieces is
    // in flight at once.
    constexpr int T = (G * D + 127) / 128;
    constexpr int hstep = 128 / D;
    float4 a[T];
#pragma unroll
    for (int t = 0; t < T; ++t) a[t] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
        const int r = i >> 5, src = i & 31;
        const int64_t bi = base(i);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const int e = 128 * t + 4 * lane;
            const int hl = (128 * t) / D;
            const bool valid = e < G * D;
            const int h = valid ? e / D : 0, dd = e - h * D;
            // every lane takes part in the shuffles; only valid lanes load
            float wi = __shfl_sync(0xffffffffu, r ? w[hl < G ? hl : 0][1] : w[hl < G ? hl : 0][0], src);
            if (hstep > 1 && hl + 1 < G) {
                const int h1 = hl + 1 < G ? hl + 1 : 0;
                const float wj = __shfl_sync(0xffffffffu, r ? w[h1][1] : w[h1][0], src);
                if (h != hl) wi = wj;
            }
            if (valid) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(&p.part_o[(bi + h) * D + dd]));
                a[t].x += wi * v.x;
                a[t].y += wi * v.y;
                a[t].z += wi * v.z;
                a[t].w += wi * v.w;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
        const int e = 128 * t + 4 * lane;
        if (e >= G * D) continue;
        const int h = e / D, dd = e - h * D;
        float ls = lsum[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh)
            if (hh == h) ls = lsum[hh];
        const float inv = (out ? oscale : 1.f) / ls;
        if (out) {
            *reinterpret_cast<uint2*>(out + h * D + dd) = make_uint2(float2_to_bf16x2(a[t].x * inv, a[t].y * inv),
                                                                     float2_to_bf16x2(a[t].z * inv, a[t].w * inv));
        } else {
            *reinterpret_cast<float4*>(&p.part_o[(base(0) + h) * D + dd]) =
                make_float4(a[t].x * inv, a[t].y * inv, a[t].z * inv, a[t].w * inv);
        }
    }
    if (!out && lane < G) {
        float mh = M[0], lh = lsum[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh)
            if (hh == lane) {
                mh = M[hh];
                lh = lsum[hh];
            }
        p.part_ml[base(0) + lane] = make_float2(mh, lh);
    }
}

// Fused append.  Every CTA writes a slice of the step's new rows, so that
// every row lands, and marks the blocks the rows go to in a hashed bitmap.
// A CTA must not read a marked block before the rows that go to it are
// there.  Two ways:
//   * local (T <= kLocalMaxTokens, the decode step's one token per
//     sequence): before loading a marked block, the producer finds the
//     tokens whose slots lie in it and writes their rows of its head group
//     itself (the same bytes the slice owner writes, so the duplicate
//     writes are harmless); no CTA waits for another, and the launch needs
//     no co-residency;
//   * barrier (more tokens): the CTAs arrive at a grid barrier (grid_bar[0]
//     counts arrivals; a cooperative launch) and a producer waits there
//     before its first marked block (a hash collision only makes it wait
//     earlier).
constexpr int kDirtyMaxTokens = 2048;  // more appended tokens: every page counts as written
constexpr int kLocalMaxTokens = 256;   // the producer warp keeps the step's slots in registers

// words * 32 is a power of two
__device__ __forceinline__ bool block_marked(const uint32_t* map, int words, int32_t blk) {
    const uint32_t bit = uint32_t(blk) & uint32_t(words * 32 - 1);
    return (map[bit >> 5] >> (bit & 31)) & 1u;
}

// Waits, in every lane of the calling warp, until all CTAs have arrived
// (bounded in time); then orders the lane's later TMA (async-proxy) reads
// after the rows they wrote.  False if it gave up or *abort was set.
__device__ __forceinline__ bool wait_rows_written(const DecodeParams& p, volatile int* abort) {
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    for (uint32_t it = 0; ld_acquire_gpu(&p.grid_bar[0]) < gridDim.x; ++it) {
        __nanosleep(32);
        if ((it & 63u) == 63u) {
            if (*abort) {
                ok = false;
                break;
            }
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                raise_error(PA_DEVERR_TIMEOUT);
                *abort = 1;
                ok = false;
                break;
            }
        }
    }
    ok = __all_sync(0xffffffffu, ok);
    fence_proxy_async_global();
    return ok;
}

// Each CTA departs once, after its last read of the arrival count; the last
// one to depart (when no CTA can still be waiting) resets the barrier.
__device__ __forceinline__ void depart_grid(const DecodeParams& p) {
    if (atomicAdd(&p.grid_bar[1], 1u) == gridDim.x - 1) {
        p.grid_bar[0] = 0;
        p.grid_bar[1] = 0;
    }
}

// Sequences whose whole context is their group's shared prefix take no
// units: their output is the merge of the prefix partials alone.  The
// calling threads (tid of nthreads) share CTA blockIdx.x's such sequences;
// they must have waited for the prefix pass.
template <int D>
__device__ __forceinline__ void prefix_only_outputs(const DecodeParams& p, int tid, int nthreads) {
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
        const SeqPages sp = seq_pages<16>(p, b, false);
        if (sp.P == 0 || sp.np != 0) continue;
        const int per = prefix_split_pages(sp.P, p.prefix_splits);
        const int nz = (sp.P + per - 1) / per;
        for (int o = tid; o < p.Hq * D; o += nthreads) {
            const int h = o / D;
            float M = -INFINITY;
            for (int z = 0; z < nz; ++z) M = fmaxf(M, __ldcg(&p.prefix_ml[(int64_t(z) * p.B + b) * p.Hq + h]).x);
            float lsum = 0.f, a = 0.f;
            for (int z = 0; z < nz; ++z) {
                const int64_t idx = (int64_t(z) * p.B + b) * p.Hq + h;
                const float2 ml = __ldcg(&p.prefix_ml[idx]);
                const float w = ml.y * exp2f(ml.x - M);
                lsum += w;
                a += w * __ldcg(&p.prefix_o[idx * D + (o - h * D)]);
            }
            p.out[int64_t(b) * p.Hq * D + o] = __float2bfloat16_rn(a / lsum);
        }
    }
}

// Local fused append, consumer side.  In a decode step token b's new row
// goes to the last page of sequence b; the CTA that reads that page does
// not need it in global memory first: the consumer warp of each kv head
// loads its head's new K and V values (bf16 caches) when the segment starts
// (lane l: values E*l .. E*l+E-1, E = D/32) and writes them over the row in
// the staged tiles (the swizzled panel layout).  The slice owner still
// writes the row to the cache.
template <int D>
struct NewRow {
    static constexpr int E = D / 32;  // values per lane
    uint32_t k[E / 2], v[E / 2];      // bf16 pairs

    __device__ __forceinline__ void load(const DecodeParams& p, int b, int g, int lane) {
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(p.k_new) + ((int64_t(b) * p.Hkv + g) * D + E * lane) / 2;
        const uint32_t* vr = reinterpret_cast<const uint32_t*>(p.v_new) + ((int64_t(b) * p.Hkv + g) * D + E * lane) / 2;
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            k[i] = __ldg(kr + i);
            v[i] = __ldg(vr + i);
        }
    }
    // Writes the row over row `off` of the staged K tile kt and V tile vt.
    __device__ __forceinline__ void patch(uint8_t* kt, uint8_t* vt, int off, int lane) const {
        const int e0 = E * lane;
        const int o = tile_off(off, e0 / 8) + (e0 % 8) * 2;
        if constexpr (E == 4) {
            *reinterpret_cast<uint2*>(kt + o) = make_uint2(k[0], k[1]);
            *reinterpret_cast<uint2*>(vt + o) = make_uint2(v[0], v[1]);
        } else {
            *reinterpret_cast<uint32_t*>(kt + o) = k[0];
            *reinterpret_cast<uint32_t*>(vt + o) = v[0];
        }
    }
};

// Local fused append: the calling warp writes the rows of every appended
// token whose slot lies in block bk, for the kv heads g0 .. g0+ng-1, into
// the cache (a bit copy, or the E4M3 encoding for fp8 caches), in token
// order.  slots: lane l holds the slots of tokens l, l+32, ...
template <int D, int BS, int EB>
__device__ __forceinline__ void write_block_rows(const DecodeParams& p, const int32_t (&slots)[kLocalMaxTokens / 32],
                                                 int32_t bk, int g0, int ng, int lane) {
    constexpr int CPR = D / 8;  // 16-byte chunks of bf16 per row
#pragma unroll
    for (int k = 0; k < kLocalMaxTokens / 32; ++k) {
        if (32 * k >= p.app_tokens) break;
        unsigned hit = __ballot_sync(0xffffffffu, slots[k] >= 0 && slots[k] / BS == bk);
        while (hit) {
            const int tl = __ffs(hit) - 1;
            hit &= hit - 1;
            const int64_t t = 32 * k + tl;
            const int32_t off = __shfl_sync(0xffffffffu, slots[k], tl) - bk * BS;
            for (int c = lane; c < ng * CPR; c += 32) {
                const int g = g0 + c / CPR, ch = c % CPR;
                const int64_t src = (t * p.Hkv + g) * CPR + ch;
                if constexpr (EB == 1) {
                    append_fp8_chunk(p.k_new, p.v_new, p.slot_mapping, reinterpret_cast<uint8_t*>(p.k_cache_w),
                                     reinterpret_cast<uint8_t*>(p.v_cache_w), p.k_scale, p.v_scale, p.Hkv, CPR, p.NB,
                                     src);
                } else {
                    const int64_t dst = ((int64_t(bk) * p.Hkv + g) * BS + off) * CPR + ch;
                    p.k_cache_w[dst] = __ldg(p.k_new + src);
                    p.v_cache_w[dst] = __ldg(p.v_new + src);
                }
            }
        }
    }
}

template <int D, int G, int BS, int R, bool DUMP, bool APPEND, template <int, int, int> class Math>
__global__ void __launch_bounds__((kDecodeWarps + 1) * 32, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    using Cfg = DecodeCfg<D, BS, R, Math<D, G, BS>::kElemBytes>;
    constexpr int NW = Cfg::NW;
    constexpr int S = Cfg::kSegSlots;
    constexpr int NT = Cfg::kThreads;
    static_assert(NW + 1 <= 16, "block reductions hold 16 warps");
    static_assert(R % Cfg::kMaxSpl == 0, "the stages of a page recur in the same slots");
    static_assert(R <= kMaxRing, "one patch flag per stage");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = smem + Cfg::kRingOff;
    SegDesc* descs = reinterpret_cast<SegDesc*>(smem + Cfg::kDescOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* empty = full + R;
    uint64_t* segfull = empty + R;
    uint64_t* segempty = segfull + S;
    Misc* misc = reinterpret_cast<Misc*>(smem + Cfg::kMiscOff);
    volatile int* abort = &misc->abort;
    uint32_t* dirty_map = reinterpret_cast<uint32_t*>(smem + Cfg::kDirtyOff);
    // a shared-prefix decode keeps half the bitmap: the rest of the area stages partials
    const int kDirtyWords = (p.num_groups > 0 ? Cfg::kDirtyBytes / 2 : Cfg::kDirtyBytes) / 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int HG = p.HG, HS = p.HS, SPL = p.SPL;
    // fused append, local: consumers write token b's new row into the staged
    // tiles of bf16 caches (for fp8 caches the encoding in the consumers cost
    // more than it saved: the producer writes the row to the cache first)
    constexpr bool kConsumerPatch = APPEND && Math<D, G, BS>::kElemBytes == 2;

    // The producer's reads that need nothing computed here start now and
    // land during the set-up and the share scan: its tensor maps, and (fused
    // append, local) the step's slots, lane l holding tokens l, l+32, ...
    constexpr int kSlotRegs = kLocalMaxTokens / 32;
    int32_t my_slots[kSlotRegs];
#pragma unroll
    for (int k = 0; k < kSlotRegs; ++k) {
        const int t = 32 * k + lane;
        my_slots[k] = (APPEND && warp == NW && p.app_local && t < p.app_tokens) ? __ldg(p.slot_mapping + t) : -1;
    }
    if (warp == NW && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
    }

    if (threadIdx.x == 0) {
        for (int r = 0; r < R; ++r) {
            mbar_init(&full[r], 1);
            mbar_init(&empty[r], uint32_t(HS));
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&segfull[s], 1);
            mbar_init(&segempty[s], uint32_t(HG));
        }
        misc->abort = 0;
        fence_mbar_init();
    }
    if (p.early_ctas > 0 && warp == 0) {
        // the longest shared prefix sets how long the prefix pass holds its
        // SMs (published to the CTA by the scan's first barrier)
        int32_t pm = 0;
        for (int i = lane; i < p.num_groups; i += 32) pm = max(pm, __ldg(p.group_prefix_pages + i));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) pm = max(pm, __shfl_xor_sync(0xffffffffu, pm, off));
        if (lane == 0) misc->pmax = pm;
    }

    // Fused append: this CTA's slice of the step's new rows (the bit copy of
    // pa::append_kernel, or the E4M3 encoding of pa::append_fp8_kernel for
    // fp8 caches).  Barrier mode: written now, then arrival at the grid
    // barrier (a written row must be visible to the TMA loads of every CTA
    // that reads its block).  Local mode: nobody waits for these writes, so
    // the consumer warps make them while the first pages are in flight.
    auto append_slice = [&](int tid, int nthreads) {
        const int64_t per = (p.app_chunks + gridDim.x - 1) / gridDim.x;
        const int64_t c0 = int64_t(blockIdx.x) * per;
        const int64_t c1 = c0 + per < p.app_chunks ? c0 + per : p.app_chunks;
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        for (int64_t idx = c0 + tid; idx < c1; idx += nthreads) {
            if constexpr (Math<D, G, BS>::kElemBytes == 1) {
                append_fp8_chunk(p.k_new, p.v_new, p.slot_mapping, reinterpret_cast<uint8_t*>(p.k_cache_w),
                                 reinterpret_cast<uint8_t*>(p.v_cache_w), p.k_scale, p.v_scale, p.Hkv, CPR, p.NB,
                                 idx);
                continue;
            }
            const int64_t t = idx / (int64_t(p.Hkv) * CPR);
            const int64_t rem = idx - t * p.Hkv * CPR;
            const int32_t slot = __ldg(p.slot_mapping + t);
            if (slot < 0) continue;
            const int64_t block = slot / BS, offset = slot - (slot / BS) * BS;
            if (block >= p.NB) {
                if (rem == 0) raise_error(PA_DEVERR_SLOT);
                continue;
            }
            const int64_t g = rem / CPR, c = rem - g * CPR;
            const int64_t dst = ((block * p.Hkv + g) * BS + offset) * CPR + c;
            p.k_cache_w[dst] = __ldg(p.k_new + idx);
            p.v_cache_w[dst] = __ldg(p.v_new + idx);
        }
    };
    // The blocks the rows go to are marked in the hashed bitmap: cleared now,
    // marked after the share scan (whose barriers order the two), read by the
    // producer after the barrier that ends the set-up.  A thread's first slot
    // is loaded now so that its latency overlaps the scan.
    int32_t first_slot = -1;
    if (APPEND) {
        for (int i = threadIdx.x; i < kDirtyWords; i += NT) dirty_map[i] = 0u;
        if (threadIdx.x == 0) misc->all_dirty = p.app_tokens > kDirtyMaxTokens;
        if (threadIdx.x < p.app_tokens) first_slot = __ldg(p.slot_mapping + threadIdx.x);
        if (!p.app_local) {
            append_slice(threadIdx.x, NT);
            fence_proxy_async_global();
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) atomicAdd(&p.grid_bar[0], 1u);
        }
    }

    // ---- the CTA's share: a scan of v_b = NG * (pages(b) + seg_weight) over
    // the sequences; sequences with no context get zero output here.  When B
    // fits in one chunk the same scan also locates the share's start. ----
    const bool one_chunk = p.B <= NT;
    long long v_mine = 0, incl_mine = 0, Wt = 0;
    SeqPages sp_mine{0, 0, 0};
    for (int base = 0; base < p.B; base += NT) {
        const int b = base + threadIdx.x;
        long long v = 0;
        if (b < p.B) {
            const SeqPages sp = seq_pages<BS>(p, b, blockIdx.x == 0);
            sp_mine = sp;
            v = (long long)(sp.np > 0 ? sp.np + p.seg_weight : 0) * p.NG;
            if (sp.L == 0 && (b % int(gridDim.x)) == int(blockIdx.x)) {
                uint4* o = reinterpret_cast<uint4*>(p.out + int64_t(b) * p.Hq * D);
                for (int i = 0; i < p.Hq * D / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
            }
        }
        long long chunk_total;
        const long long incl = Wt + block_incl_scan<NT>(v, misc->red, chunk_total);  // first call also
        Wt += chunk_total;                                                          // publishes mbar init
        v_mine = v;
        incl_mine = incl;
    }
    if (APPEND && p.app_tokens <= kDirtyMaxTokens) {
        auto mark = [&](int32_t slot) {
            if (slot < 0) return;
            const uint32_t bit = uint32_t(slot / BS) & uint32_t(kDirtyWords * 32 - 1);
            atomicOr(&dirty_map[bit >> 5], 1u << (bit & 31));
        };
        mark(first_slot);
        for (int t = threadIdx.x + NT; t < p.app_tokens; t += NT) mark(__ldg(p.slot_mapping + t));
    }
    // A decode launched right after prefix_kernel (programmatic dependent
    // launch) has done the set-up above meanwhile; the prefix partials and
    // the rows that kernel appended are read only after this wait (a no-op
    // for an ordinary launch).
    if (!p.defer_dep) asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t want = (Wt + p.min_pages - 1) / p.min_pages;
    const int64_t grid_eff = want < int64_t(gridDim.x) ? want : int64_t(gridDim.x);
    if (Wt == 0 || int64_t(blockIdx.x) >= grid_eff) {  // no share: read no page
        if (APPEND && p.app_local) append_slice(threadIdx.x, NT);
        if (APPEND && !p.app_local && threadIdx.x == 0) depart_grid(p);
        if (p.num_groups > 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            prefix_only_outputs<D>(p, threadIdx.x, NT);
        }
        return;
    }
    // the early CTAs' extra units: what one CTA streams while the prefix pass runs
    int64_t want_x = 0;
    if (p.early_ctas > 0 && misc->pmax > 0) {
        const int64_t ns = p.early_ns + int64_t(p.early_ns_per_page) * prefix_split_pages(misc->pmax, p.prefix_splits);
        want_x = ns * p.early_units_per_ms / 1000000;
    }
    const Split split = make_split(Wt, grid_eff, p.early_ctas, want_x, p.min_pages);
    const int64_t p_start = split.start(blockIdx.x);
    const int64_t p_end = split.start(int64_t(blockIdx.x) + 1);

    // ---- the sequence where the share starts (with its page counts, so the
    // producer starts without reading them again) ----
    auto locate = [&](int b, long long v, long long incl, const SeqPages& sp) {
        const long long lo = incl - v;
        if (v > 0 && lo <= p_start && p_start < incl) {
            misc->b0 = b;
            misc->L0 = sp.L;
            misc->P0 = sp.P;
            misc->np0 = sp.np;
            misc->pre0 = lo;
        }
    };
    if (one_chunk) {
        locate(threadIdx.x, v_mine, incl_mine, sp_mine);
    } else {
        long long carry = 0;
        for (int base = 0; base < p.B; base += NT) {
            const int b = base + threadIdx.x;
            long long v = 0;
            SeqPages sp{0, 0, 0};
            if (b < p.B) {
                sp = seq_pages<BS>(p, b, false);
                v = (long long)(sp.np > 0 ? sp.np + p.seg_weight : 0) * p.NG;
            }
            long long chunk_total;
            const long long incl = carry + block_incl_scan<NT>(v, misc->red, chunk_total);
            locate(b, v, incl, sp);
            carry += chunk_total;
        }
    }
    __syncthreads();

    if (warp == NW) {
        // ======================= producer warp =======================
        uint32_t stage_i = 0, seg_i = 0;
        constexpr int C = R < 32 ? R : 32;
        bool ok = true;
        bool rows_ready = !APPEND;  // fused append, barrier: every CTA's rows are visible
        const uint64_t pol = PA_EVICT_FIRST ? policy_evict_first() : policy_evict_normal();
        const uint32_t stage_tx = uint32_t(2 * HS * Cfg::kTile);

        // walk the (b, hg) whose units meet the share [p_start, p_end)
        int b = misc->b0;
        SeqPages sp{misc->L0, misc->P0, misc->np0};
        int32_t Lb = sp.L, Pb = sp.P, np = sp.np;  // the line holds b's pages Pb .. Pb+np-1
        int64_t unit = np + p.seg_weight;
        int hg = int((p_start - misc->pre0) / unit);
        int64_t u0 = misc->pre0 + int64_t(hg) * unit;  // line position of (b, hg)'s first page
        while (ok && u0 < p_end) {
            const int64_t lo = p_start > u0 ? p_start : u0;
            const int64_t hi = p_end < u0 + np ? p_end : u0 + np;
            if (lo < hi) {
                const int j = Pb + int(lo - u0);  // first page of the segment in b's table
                const int npg = int(hi - lo);
                if (lane == 0) {
                    const int s = seg_i % S;
                    if (seg_i >= S) ok = mbar_wait(&segempty[s], ((seg_i / S) - 1) & 1, abort);
                    if (ok) {
                        SegDesc& d = descs[s];
                        d.b = b;
                        d.hg = hg;
                        d.j0 = j;
                        d.npg = npg;
                        d.L = Lb;
                        d.k0 = split.owner(u0);
                        d.k1 = split.owner(u0 + np - 1);
                        d.P = Pb;
                        mbar_arrive(&segfull[s]);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                // one lane per stage: HS heads' K tiles, then their V tiles
                const int32_t* bt = p.block_tables + int64_t(b) * p.M + j;
                const int tile0 = hg * HG;
                const int nst = npg * SPL;
                for (int c0 = 0; ok && c0 < nst; c0 += C) {
                    const int n = (nst - c0) < C ? (nst - c0) : C;
                    bool lane_ok = true;
                    int32_t blk = 0;
                    if (lane < n) {
                        blk = __ldg(bt + ((c0 + lane) >> p.SPL_LOG));
                        if (blk < 0 || blk >= p.NB) {
                            raise_error(PA_DEVERR_BLOCK_ID);
                            blk = 0;
                        }
                    }
                    bool patch_page = false;  // this lane's stage: the consumers write the new row
                    if (APPEND && p.app_local) {
                        // Each marked page of the batch (its first stage's lane stands
                        // for it): when its only new row is token b's, at the last
                        // position of b, in b's last page, the consumers write that row
                        // into the staged tiles; otherwise the new rows are written to
                        // the cache here before the page is loaded.
                        const bool marked = lane < n && ((c0 + lane) & (SPL - 1)) == 0 &&
                                            block_marked(dirty_map, kDirtyWords, blk);
                        unsigned pages_hit = __ballot_sync(0xffffffffu, marked);
                        unsigned by_consumers = 0u;
                        bool wrote = false;
                        while (pages_hit) {
                            const int src = __ffs(pages_hit) - 1;
                            pages_hit &= pages_hit - 1;
                            const int32_t bk = __shfl_sync(0xffffffffu, blk, src);
                            int cnt = 0, t_first = -1;
                            int32_t s_first = 0;
#pragma unroll
                            for (int k = 0; k < kLocalMaxTokens / 32; ++k) {
                                const unsigned h = __ballot_sync(0xffffffffu, my_slots[k] >= 0 && my_slots[k] / BS == bk);
                                if (h && t_first < 0) {
                                    const int tl = __ffs(h) - 1;
                                    t_first = 32 * k + tl;
                                    s_first = __shfl_sync(0xffffffffu, my_slots[k], tl);
                                }
                                cnt += __popc(h);
                            }
                            const int page = j + ((c0 + src) >> p.SPL_LOG);
                            if (kConsumerPatch && cnt == 1 && t_first == b && page == (Lb - 1) / BS &&
                                s_first % BS == (Lb - 1) % BS) {
                                by_consumers |= 1u << src;
                            } else if (cnt > 0) {
                                write_block_rows<D, BS, Math<D, G, BS>::kElemBytes>(p, my_slots, bk, tile0, HG,
                                                                                     lane);
                                wrote = true;
                            }
                        }
                        if (wrote) {
                            fence_proxy_async_global();
                            __syncwarp();
                            fence_proxy_async_global();
                        }
                        // every stage of a page follows its first stage's lane
                        const int lead = lane & ~(SPL - 1);
                        patch_page = (by_consumers >> lead) & 1u;
                    } else if (APPEND && !rows_ready) {
                        const bool marked =
                            lane < n && (misc->all_dirty || block_marked(dirty_map, kDirtyWords, blk));
                        if (__any_sync(0xffffffffu, marked)) {
                            rows_ready = true;
                            if (!wait_rows_written(p, abort)) {
                                ok = false;
                                break;
                            }
                        }
                    }
                    if (lane < n) {
                        const int x = c0 + lane;
                        const int sub = x & (SPL - 1);
                        const uint32_t i = stage_i + x;
                        const int slot = int(i % R);
                        const uint32_t use = i / R;
                        if (use > 0) lane_ok = mbar_wait(&empty[slot], (use - 1) & 1, abort);
                        if (lane_ok) {
                            uint8_t* st = ring + slot * Cfg::kStage;
                            if (APPEND) misc->patch[slot] = patch_page ? 1 : 0;
                            mbar_arrive_expect_tx(&full[slot], stage_tx);
                            const int tile = blk * p.Hkv + tile0 + sub * HS;
                            tma_load_4d(st, &p.tmap_k, 0, 0, 0, tile, &full[slot], pol);
                            tma_load_4d(st + Cfg::kStageK, &p.tmap_v, 0, 0, 0, tile, &full[slot], pol);
                        }
                    }
                    ok = __all_sync(0xffffffffu, lane_ok);
                }
                stage_i += nst;
                ++seg_i;
            }
            // next (b, hg) on the line (sequences without own pages take no units)
            u0 += unit;
            if (u0 < p_end && ++hg == p.NG) {
                hg = 0;
                do {
                    ++b;
                    sp = seq_pages<BS>(p, b, false);
                } while (sp.np == 0);
                Lb = sp.L;
                Pb = sp.P;
                np = sp.np;
                unit = np + p.seg_weight;
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
            const uint32_t last = stage_i + C;
            for (uint32_t i = (last > R ? last - R : 0); i < last; ++i)
                mbar_wait(&full[i % R], (i / R) & 1, nullptr, 20000000ull);
        }
        if (APPEND && !p.app_local && lane == 0) depart_grid(p);
        if (p.num_groups > 0) {  // after this warp's last copy: the prefix-only sequences
            asm volatile("griddepcontrol.wait;" ::: "memory");
            prefix_only_outputs<D>(p, lane, 32);
        }
        return;
    }
    if (APPEND && p.app_local) append_slice(threadIdx.x, NW * 32);  // warps 0 .. NW-1
    if (warp >= HG) return;

    // ========================= consumer warps =========================
    using MathT = Math<D, G, BS>;
    MathT st;
    // this warp's staging of prefix range partials: per range G*D floats of
    // output, then G (max, sum) pairs; 16-byte copies of whole pairs need G even
    constexpr int kRangeBytes = G * D * 4 + ((G * 8 + 15) / 16) * 16;
    constexpr int kStageWarpBytes = ((Cfg::kAreaBytes - Cfg::kDirtyBytes / 2) / NW) / 16 * 16;
    constexpr int kStagedRanges = (G % 2 == 0) ? kStageWarpBytes / kRangeBytes : 0;
    uint8_t* stage_area = smem + Cfg::kDirtyOff + Cfg::kDirtyBytes / 2 + warp * kStageWarpBytes;
    bool dep_done = !p.defer_dep;  // this warp has waited for the prefix pass
    uint32_t stage_base = 0, seg_i = 0;
    const int64_t hgG = int64_t(HG) * G;  // query heads of one partial slot
    const int sub = warp / HS;              // this warp's stage within a page
    const int pos = warp - sub * HS;        // and its tile within that stage

    while (true) {
        const int s = seg_i % S;
        if (!mbar_wait(&segfull[s], (seg_i / S) & 1, abort)) return;
        const SegDesc d = descs[s];
        __syncwarp();
        if (lane == 0) mbar_arrive(&segempty[s]);
        if (d.npg == 0) break;
        const int g = d.hg * HG + warp;  // this warp's kv head
        const int64_t row = int64_t(d.b) * p.Hq + int64_t(g) * G;  // its first query head
        st.load_q_global(p.q + row * (D * 2), lane, p.k_scale ? p.qscale * __ldg(p.k_scale + g) : p.qscale);
        st.oscale = p.v_scale ? __ldg(p.v_scale + g) : 1.f;
        st.reset();
        // The piece that starts at b's first own page carries the shared
        // prefix: the partials of its nz prefix key ranges are folded in after
        // the pages.  When they fit, all of them are copied now (cp.async)
        // into this warp's staging area and folded from shared memory, so the
        // copies overlap the pages; otherwise range 0 is loaded into
        // registers now and the others are read after the pages.
        const int nz = (d.P > 0 && d.j0 == d.P)
                           ? (d.P + prefix_split_pages(d.P, p.prefix_splits) - 1) /
                                 prefix_split_pages(d.P, p.prefix_splits)
                           : 0;
        const bool staged = nz > 0 && nz <= kStagedRanges;
        typename MathT::Piece piece;
        auto stage_ranges = [&]() {
            for (int z = 0; z < nz; ++z) {
                const int64_t idx = int64_t(z) * p.B * p.Hq + row;
                uint8_t* dst = stage_area + z * kRangeBytes;
                const uint8_t* so = reinterpret_cast<const uint8_t*>(p.prefix_o + idx * D);
                for (int c = lane; c < G * D / 4; c += 32) cp_async16(dst + 16 * c, so + 16 * c);
                const uint8_t* sml = reinterpret_cast<const uint8_t*>(p.prefix_ml + idx);
                if (lane < G / 2) cp_async16(dst + G * D * 4 + 16 * lane, sml + 16 * lane);
            }
            cp_async_commit();
        };
        // the partials exist once the prefix pass is complete: a warp that has
        // waited for it once fetches them now, otherwise after the pages
        const bool early = nz > 0 && dep_done;
        if (early && staged) stage_ranges();
        else if (early) st.piece_load(piece, p.prefix_o + row * D, p.prefix_ml + row, lane);

        // fused append, local: token b's new row of this warp's head, written
        // over the staged tiles of the stages the producer flags
        // (only the segment's last page, when it is b's last page, can carry
        // the row: the flag is read there alone, so other pages pay nothing)
        NewRow<D> nrow;
        int patch_k = -1;  // the page of this segment that may take the row
        if constexpr (kConsumerPatch) {
            if (p.app_local && (d.j0 + d.npg) * BS >= d.L && d.b < p.app_tokens) {
                nrow.load(p, d.b, g, lane);
                patch_k = d.npg - 1;
            }
        }

        // (R is a multiple of SPL, so the stages of each warp recur in the
        // same slots and every parity wait is exact)
        if constexpr (MathT::kPairPages) {
            // two pages per softmax step (one stage per page: SPL == 1 here)
            for (int k = 0; k < d.npg; k += 2) {
                const uint32_t i0 = stage_base + uint32_t(k), i1 = i0 + 1;
                const bool two = k + 1 < d.npg;
                const int slot0 = int(i0 % R), slot1 = int(i1 % R);
                if (!mbar_wait(&full[slot0], (i0 / R) & 1, abort)) return;
                if (two && !mbar_wait(&full[slot1], (i1 / R) & 1, abort)) return;
                const uint8_t* kt0 = ring + slot0 * Cfg::kStage + pos * Cfg::kTile;
                const uint8_t* kt1 = two ? ring + slot1 * Cfg::kStage + pos * Cfg::kTile : kt0;
                const int nr0 = d.L - (d.j0 + k) * BS, nr1 = d.L - (d.j0 + k + 1) * BS;
                const int nv0 = nr0 < BS ? nr0 : BS;
                const int nv1 = two ? (nr1 < BS ? nr1 : BS) : 0;

                st.page2(kt0, kt0 + Cfg::kStageK, nv0, kt1, kt1 + Cfg::kStageK, nv1, lane);
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&empty[slot0]);
                    if (two) mbar_arrive(&empty[slot1]);
                }
            }
        } else
        for (int k = 0; k < d.npg; ++k) {
            const uint32_t i = stage_base + uint32_t(k * SPL + sub);
            const int slot = int(i % R);
            if (!mbar_wait(&full[slot], (i / R) & 1, abort)) return;
            uint8_t* kt = ring + slot * Cfg::kStage + pos * Cfg::kTile;
            uint8_t* vt = kt + Cfg::kStageK;
            const int nv_raw = d.L - (d.j0 + k) * BS;
            const int nv = nv_raw < BS ? nv_raw : BS;
            bool wrote = false;
            if constexpr (kConsumerPatch) {
                if (k == patch_k && misc->patch[slot]) {
                    nrow.patch(kt, vt, (d.L - 1) % BS, lane);
                    wrote = true;
                }
            }
            if (MathT::kZeroMaskedV && nv < BS) {
                // rows past the context may hold anything (NaN included): clear
                // them in this head's V tile so that 0 * row stays 0 in the tensor core
                constexpr int NPANEL = D / 64;
                const int per_panel = (BS - nv) * 8;  // 16-byte chunks
                for (int x = lane; x < NPANEL * per_panel; x += 32) {
                    const int pn = x / per_panel, rem = x - pn * per_panel;
                    const int t = nv + (rem >> 3), cch = rem & 7;
                    *reinterpret_cast<uint4*>(vt + pn * Cfg::kPanel + t * 128 + cch * 16) = make_uint4(0, 0, 0, 0);
                }
                wrote = true;
            }
            if (wrote) {  // before the page math, and before the stage is refilled by TMA
                __syncwarp();
                fence_proxy_async_smem();
            }
            st.page(kt, vt, nv, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        stage_base += uint32_t(d.npg * SPL);
        if (nz > 0 && !early) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            dep_done = true;
            if (staged) stage_ranges();
            else st.piece_load(piece, p.prefix_o + row * D, p.prefix_ml + row, lane);
        }
        if (staged) {
            cp_async_wait_all();
            __syncwarp();
            for (int z = 0; z < nz; ++z) {
                const uint8_t* src = stage_area + z * kRangeBytes;
                st.template absorb<true>(reinterpret_cast<const float*>(src),
                                         reinterpret_cast<const float2*>(src + G * D * 4), lane);
            }
            __syncwarp();  // read before the next segment's copies land
        } else if (nz > 0) {
            st.piece_absorb(piece, lane);
            for (int z = 1; z < nz; ++z) {
                const int64_t idx = int64_t(z) * p.B * p.Hq + row;
                st.absorb(p.prefix_o + idx * D, p.prefix_ml + idx, lane);
            }
        }

        // ---- segment end: this warp's (b, g) result ----
        const bool whole = d.k0 == d.k1;
        const int nk = d.k1 - d.k0 + 1;
        const int leaf = int(blockIdx.x) - d.k0;
        int32_t* top = p.counters + int64_t(d.b) * p.Hkv + g;
        if (!DUMP && !whole && nk <= kFastMergePieces) {
            // ticket first; the second piece to finish merges the first one's
            // published partial with its own registers, in leaf order
            if (ticket(top, nk, lane)) {
                const int64_t sl = leaf_slot(d.k0, 1 - leaf);
                const int* flag = p.slot_sync + sl * HG + warp;
                const uint64_t t0 = globaltimer_ns();
                for (uint32_t it = 0; ld_acquire_gpu(flag) == 0; ++it) {  // set right after its ticket
                    __nanosleep(32);
                    if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) {
                        raise_error(PA_DEVERR_TIMEOUT);
                        break;
                    }
                }
                __syncwarp();
                const int64_t ps = sl * hgG + int64_t(warp) * G;
                typename MathT::Piece other;
                st.piece_load(other, p.part_o + ps * D, p.part_ml + ps, lane);
                st.finish();
                st.store_merged2(other, leaf == 0, p.out + row * D, lane);
                __syncwarp();
                if (lane == 0) {
                    p.slot_sync[sl * HG + warp] = 0;
                    *top = 0;
                }
            } else {
                const int64_t ps = leaf_slot(d.k0, leaf) * hgG + int64_t(warp) * G;
                st.finish();
                st.store_partial(p.part_o + ps * D, p.part_ml + ps, nullptr, nullptr, lane);
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(p.slot_sync + leaf_slot(d.k0, leaf) * HG + warp, 1);
            }
            ++seg_i;
            continue;
        }
        st.finish();
        if (DUMP) {
            int di = 0;
            if (lane == 0) di = atomicAdd(p.seg_count, 1);
            di = __shfl_sync(0xffffffffu, di, 0);
            if (di < p.dump_capacity) {
                st.store_partial(p.seg_o + int64_t(di) * G * D, nullptr, p.seg_m + int64_t(di) * G,
                                 p.seg_l + int64_t(di) * G, lane);
                if (lane == 0) {
                    int32_t* mt = p.seg_meta + int64_t(di) * 4;
                    mt[0] = d.b;
                    mt[1] = g;
                    mt[2] = d.j0 * BS;
                    const int t1 = (d.j0 + d.npg) * BS;
                    mt[3] = t1 < d.L ? t1 : d.L;
                }
            }
        }
        if (whole) {
            st.store_out(p.out + row * D, lane);
        } else {
            // ---- split-KV: the last CTA to finish a piece of (b, g) merges.
            // Partial slot: the piece of the CTA that owns the segment's first
            // page goes to slot 1 (it ends that CTA's share), any other piece
            // to slot 0 (it starts its CTA's share): one of each per CTA. ----
            const int my_slot = int(blockIdx.x) == d.k0 ? 1 : 0;
            const int64_t ps = (int64_t(blockIdx.x) * 2 + my_slot) * hgG + int64_t(warp) * G;
            st.store_partial(p.part_o + ps * D, p.part_ml + ps, nullptr, nullptr, lane);
            __threadfence();
            __syncwarp();
            if (nk <= kMergeFanIn) {
                if (ticket(top, nk, lane)) {
                    merge_pieces<D, G>(p, d.k0, 0, 1, nk, HG, warp, lane, p.out + row * D, st.oscale);
                    if (lane == 0) *top = 0;
                }
            } else {
                const int first = leaf - leaf % kMergeFanIn;
                const int runs = (nk + kMergeFanIn - 1) / kMergeFanIn;
                const int in_run = nk - first < kMergeFanIn ? nk - first : kMergeFanIn;
                int32_t* gc = p.slot_sync + (int64_t(d.k0 + first) * 2 + (first == 0 ? 1 : 0)) * HG + warp;
                if (ticket(gc, in_run, lane)) {
                    // this run's pieces -> the partial slot of its first piece
                    merge_pieces<D, G>(p, d.k0, first, 1, in_run, HG, warp, lane, nullptr);
                    if (lane == 0) *gc = 0;
                    __threadfence();
                    __syncwarp();
                    if (ticket(top, runs, lane)) {
                        merge_pieces<D, G>(p, d.k0, 0, kMergeFanIn, runs, HG, warp, lane, p.out + row * D, st.oscale);
                        if (lane == 0) *top = 0;
                    }
                }
            }
        }
        ++seg_i;
    }
}

}  // namespace pa
