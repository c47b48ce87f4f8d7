// Paged decode attention kernels for sm_100a.
//
// pa_decode_kernel: by default one CTA per (sequence, kv head, partition);
// with balanced ranges, one wave of CTAs that each walk an equal contiguous
// share of all (sequence, kv head, page) work, one unit segment at a time
// (see DecodeParams::balanced).  Within a segment, four warps (two for 16 KiB
// stages), each an independent producer/consumer pipeline over its share of
// the segment's stages (stages w, w+4, w+8, ... of the segment).  A stage is
// one page, or two consecutive pages when pages are small (pair_pages).
//   * Lane 0 of a warp reads the block table (the page table of
//     "Why PagedAttention was retired", section 1), widens the physical id to
//     64 bits, and moves the whole (block, kv head) K page and V page --
//     each one contiguous run of head_size*block_size elements in the cache
//     layouts of section 2 -- into a shared-memory stage with 1-D bulk async
//     copies (two per page) that complete on the stage's mbarrier.
//   * The warp consumes a landed page once: S = Q K^T on the tensor cores
//     (m16n8k16, heads on M, tokens on N, head dim on K), online softmax in
//     fp32 registers (row max/sum over the quad by shuffles), then
//     O^T += V^T P^T (head dim on M, heads on N, tokens on K).  K and V are
//     each read from HBM exactly once -- the single traversal that replaces
//     the legacy kernel's two passes (section 3 of the same page).
//   * FP8 e4m3 pages are converted in registers (exact e4m3 -> f16) right
//     before the MMA; k_scale folds into the logit scale and v_scale into the
//     output, so the conversion needs no multiply (section 4 of the page).
//   * The warps' (max, sum, acc) are merged in shared memory; the CTA
//     writes bf16 out directly, or, when the unit is split over several
//     partitions (or cut at a balanced range's end), an fp32 partial plus its
//     (max, sum) for pa_combine_kernel (the exp_sums / max_logits /
//     tmp_output roles of the partitioned variant in the PR #47361 benchmark
//     snippet).
//
// Every mbarrier wait is bounded (~2 s); on give-up the warp drains its copies
// in flight (bounded too), ORs PA_DEV_WAIT_TIMEOUT into the status word and
// finishes without touching further pages.
#pragma once

#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "pa_ptx.cuh"

namespace pa {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kFull = 0xffffffffu;

constexpr uint32_t kDevBadBlock = 0x1u;
constexpr uint32_t kDevSeqLen = 0x2u;
constexpr uint32_t kDevTimeout = 0x4u;
constexpr uint32_t kDevPrefix = 0x8u;

struct DecodeParams {
    __nv_bfloat16* out;       // [S, Hq, D]
    const uint16_t* q;        // bf16 bits [S, Hq, D]
    const uint8_t* kc;        // K cache bytes
    const uint8_t* vc;        // V cache bytes
    const int32_t* bt;        // [S, max_blocks]
    const int32_t* seq_lens;  // [S]
    const float* k_scale;     // fp8 only
    const float* v_scale;     // fp8 only
    float* ws_o;              // [S, Hq, P, D]   (P > 1)
    float* ws_m;              // [S, Hq, P]      running max, log2 domain
    float* ws_l;              // [S, Hq, P]      running sum
    uint32_t* status;         // sticky status word
    int S, Hq, Hk, G;
    int max_blocks;
    int P;   // partitions per (seq, kv head) over its own pages
    int PP;  // pages per partition
    int stages;
    long long num_blocks;
    float scale_log2;  // scale * log2(e)
    // Shared-prefix (cascade) decode: the first prefix_pages logical blocks are
    // the same physical blocks in every row of the block table.  They are
    // streamed once per group of 16 query rows (all sequences' heads of one kv
    // head) by the first prefix_units CTAs; per-sequence CTAs start after them.
    int prefix_pages;         // 0: no shared prefix
    int prefix_parts;         // partitions of the prefix
    int prefix_groups;        // 16-row groups of the S*G query rows of a kv head
    // Prefix CTAs per (kv head, partition): with prefix_shared (at least W
    // groups), one per W groups, streaming each page once through a ring
    // shared by its warps (prefix_shared_ring); otherwise one per group, its
    // warps splitting the pages like a sequence's unit.
    int prefix_shared;
    int prefix_cta_groups;
    long long prefix_units;   // Hk * prefix_cta_groups * prefix_parts
    int P_total;              // partial slots per (seq, q head): prefix_parts + P
    const float* alibi;       // [Hq] ALiBi slopes, or nullptr
    // Failure-path test hook: each page's mbarrier expects stall_tx_bytes more
    // than its copies deliver, so every wait runs out after wait_limit_ns.
    int stall_tx_bytes;
    unsigned long long wait_limit_ns;
    // Longest first: per-sequence CTAs take sequences in order of decreasing
    // length (ties by index), ranked by every CTA from seq_lens (num_seqs <= 256).
    int longest_first;
    // Balanced ranges (no shared prefix): the grid's CTAs take equal contiguous
    // shares of all pages in (sequence, kv head, page) order, and each walks
    // its share one unit segment at a time.  A segment that is a whole unit
    // writes `out`; a cut one writes slot 2 c + k of CTA c (k = 0: the first
    // segment of its range, 1: the last), rows of G query heads, for
    // pa_combine_kernel.  CTA 0 leaves the per-sequence page prefix and the
    // pages per CTA in br_scan[0 .. S + 1] for the combine.
    int balanced;
    int* br_scan;
    // Split tail (the partitioned schedule where units are not split): the
    // first n_full per-sequence units run whole; each remaining unit is cut
    // into tail_P partitions of tail_PP pages, whose CTAs come after every
    // whole unit's.  Tail unit t = unit - n_full writes its partials at rows
    // (t * G + g) * tail_P + part of ws_o / ws_m / ws_l.
    long long n_full;
    int tail_P, tail_PP;
    // The split tail's merge counts: each CTA of tail unit t counts itself in
    // at merge_cnt[t]; the unit's last CTA merges its rows into out and sets
    // the count back to 0 (counts are 0 between calls).
    unsigned int* merge_cnt;
};

// Bytes of shared memory the final merge needs (it overlays the page stages).
template <int D, int NH, int W>
constexpr int merge_smem_bytes() {
    return (W * NH * 8 * (D + 4) + 2 * W * 16) * 4;
}

// Consumer warps per decode CTA.  Pages of 16 KiB stages (bf16, head size
// 128, block size 32) get two warps so that three CTAs still fit on an SM;
// smaller pages get four.
constexpr int decode_warps(long long stage_bytes) { return stage_bytes >= 16384 ? 2 : 4; }

// Whether a stage holds two 16-token pages: e4m3 pages, and bf16 pages of
// head size 64 (2 KiB at most).  Pairs double a warp's bytes in flight at
// the same warps per SM; measured on B200, 4 KiB pages stream faster than
// 2 KiB ones (bf16 pages of head size 128 are 4 KiB already).
template <int D, int B, bool FP8, bool F8MMA>
constexpr bool pair_pages() {
    return B == 16 && (FP8 || D == 64);
}

template <int D, int B, bool FP8>
constexpr int decode_warps() {
    return decode_warps(2LL * D * B * (FP8 ? 1 : 2));
}

// One warp's attention state over a run of pages of one unit, and the work
// on one landed page: the query as MMA operands, the running (max, sum) of
// its rows and the O^T accumulator, all in registers.  Rows are query heads
// 8r + gq of the unit (NH blocks of 8 MMA rows); the page body is shared by
// every schedule of the decode kernel.
template <int D, int B, bool FP8, int NH, bool F8MMA>
struct WarpAttn {
    static constexpr int ELEM = FP8 ? 1 : 2;
    static constexpr int K32 = D / 32;  // 32-wide k-steps over the head dim (e4m3 MMA)
    static constexpr int PAGE = D * B * ELEM;  // one K (or V) page of one kv head
    static constexpr bool PAIR = pair_pages<D, B, FP8, F8MMA>();
    static constexpr int NPG = PAIR ? 2 : 1;  // logical pages per stage
    static constexpr int BT = B * NPG;        // tokens per stage
    static constexpr int NT = BT / 8;  // 8-token n-tiles per stage (QK)
    static constexpr int KT = D / 16;  // 16-wide k-tiles over the head dim (QK)
    static constexpr int MT = D / 16;  // 16-row m-tiles over the head dim (PV)
    static constexpr int KK = BT / 16; // 16-token k-tiles per stage (PV)
    static constexpr int CHUNK = B * 16;  // bytes of one 16-byte column group of a K page

    int lane, gq, cq;
    int src0, src1;
    bool hi_half;
    uint32_t qa[F8MMA ? 1 : KT][4];
    uint32_t qa8[F8MMA ? K32 : 1][2][4];  // e4m3 MMAs: [k-step][hi, lo][regs]
    float qk_mul, out_mul;
    float slope2[NH];  // ALiBi slope of each row in log2 units (0 without ALiBi)
    float m_run[NH], l_run[NH];
    float acc[MT][NH][4];

    __device__ __forceinline__ explicit WarpAttn(int lane_) {
        lane = lane_;
        gq = lane >> 2;  // fragment row group
        cq = lane & 3;   // thread in quad
        const int quad0 = lane & ~3;
        src0 = quad0 | ((2 * cq) & 3);
        src1 = quad0 | ((2 * cq + 1) & 3);
        hi_half = cq >= 2;
    }

    uint32_t qraw[2][KT][2];  // raw query words until finish_query

    // Start loading the query rows row_of(8r + gq) (-1: none) in the order
    // the fragments use them; finish_query turns them into MMA operands.
    template <class RowFn>
    __device__ __forceinline__ void fetch_query(const uint16_t* q, RowFn row_of) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const long long qr = (r < NH) ? row_of(8 * r + gq) : -1;
            const bool ok = qr >= 0;
            const uint16_t* qrow = q + (ok ? qr : 0) * D;
#pragma unroll
            for (int kt = 0; kt < KT; ++kt) {
                uint32_t w0 = 0, w1 = 0;
                if (ok) {
                    if constexpr (!FP8) {
                        const unsigned int* qw = reinterpret_cast<const unsigned int*>(qrow);
                        w0 = __ldg(qw + 8 * kt + cq);
                        w1 = __ldg(qw + 8 * kt + 4 + cq);
                    } else {
                        const uint2 w =
                            __ldg(reinterpret_cast<const uint2*>(qrow + 16 * kt + 4 * cq));
                        w0 = w.x;
                        w1 = w.y;
                    }
                }
                qraw[r][kt][0] = w0;
                qraw[r][kt][1] = w1;
            }
        }
    }

    __device__ __forceinline__ void finish_query(float scale_log2, float k_scale, float v_scale) {
        load_q(qraw, scale_log2, k_scale, v_scale);
    }

    // ALiBi: the logit of token t gains slope * (t - (T - 1)); slopes of rows
    // row_of(8r + gq), kept in log2 units (0 without ALiBi).
    template <class RowFn>
    __device__ __forceinline__ void set_alibi(const float* alibi, int Hq, RowFn row_of) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            const long long qr = row_of(8 * r + gq);
            slope2[r] = (alibi && qr >= 0) ? __ldg(alibi + qr % Hq) * 1.4426950408889634f : 0.f;
        }
    }

    // Q fragments (A operand of S = Q K^T; rows = heads 8r + gq) from the raw
    // bf16 query words of rows 8r + gq, in the order the fragments use, and
    // the logit multiplier (log2 domain) and output multiplier that go with them.
    __device__ __forceinline__ void load_q(const uint32_t (&qraw)[2][KT][2], float scale_log2,
                                           float k_scale, float v_scale) {
        qk_mul = scale_log2;
        out_mul = 1.f;
        if constexpr (F8MMA) {
            // e4m3 operands: q is scaled by 2^e so that max|q| 2^e < 256, then
            // split into hi + lo e4m3 codes (about 2^-8 relative together); both
            // halves multiply the same K bytes, so one accumulator takes both.
            // Natural d order: register i holds d = 32 jp + 16 (i >> 1) + 4 cq + 0..3.
            float amax = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    const uint32_t w0 = qraw[r][kt][0], w1 = qraw[r][kt][1];
                    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(w0)), fabsf(bf16_hi(w0))),
                                             fmaxf(fabsf(bf16_lo(w1)), fabsf(bf16_hi(w1)))));
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
            int e = 0;
            if (amax > 0.f && amax < INFINITY)
                e = 7 - (static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127);
            e = max(-100, min(100, e));
            const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
            const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
            for (int jp = 0; jp < K32; ++jp)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = i & 1, kt = 2 * jp + (i >> 1);
                    if (r >= NH) {  // rows 8..15 unused: zero codes
                        qa8[jp][0][i] = 0u;
                        qa8[jp][1][i] = 0u;
                        continue;
                    }
                    const uint32_t w0 = qraw[r][kt][0], w1 = qraw[r][kt][1];
                    float unused;
                    const uint32_t a = split_e4m3x2(bf16_lo(w0) * up, bf16_hi(w0) * up, &unused);
                    const uint32_t b = split_e4m3x2(bf16_lo(w1) * up, bf16_hi(w1) * up, &unused);
                    qa8[jp][0][i] = __byte_perm(a, b, 0x5410);  // hi codes of d .. d+3
                    qa8[jp][1][i] = __byte_perm(a, b, 0x7632);  // lo codes
                }
            qk_mul = scale_log2 * k_scale * down;
            out_mul = v_scale;
        } else if constexpr (!FP8) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    qa[kt][r] = qraw[r][kt][0];
                    qa[kt][r + 2] = qraw[r][kt][1];
                }
        } else {
            // f16 operands: q is scaled by 2^-e so that max|q| < 2^15 (f16 range);
            // 2^e goes back into the logit multiplier.  Within each 16-wide chunk the
            // k order is permuted to match the e4m3 byte order delivered by ldmatrix:
            // k = 2c,2c+1 <-> d = 4c,4c+1 and k = 2c+8,2c+9 <-> d = 4c+2,4c+3.
            float amax = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    const uint32_t w0 = qraw[r][kt][0], w1 = qraw[r][kt][1];
                    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(w0)), fabsf(bf16_hi(w0))),
                                             fmaxf(fabsf(bf16_lo(w1)), fabsf(bf16_hi(w1)))));
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
            int ex = 0;
            if (amax > 0.f && amax < INFINITY)
                ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xff) - 127;
            const int e = ex > 14 ? ex - 14 : 0;
            const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
            const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    const uint32_t w0 = qraw[r][kt][0], w1 = qraw[r][kt][1];
                    qa[kt][r] = pack_f16x2(bf16_lo(w0) * down, bf16_hi(w0) * down);
                    qa[kt][r + 2] = pack_f16x2(bf16_lo(w1) * down, bf16_hi(w1) * down);
                }
            qk_mul = scale_log2 * k_scale * up;
            out_mul = v_scale;
        }
    }

    // Sum each row's l over its quad, so every thread of a quad holds its
    // row's total (before the state leaves the warp).
    __device__ __forceinline__ void reduce_l() {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            l_run[r] += __shfl_xor_sync(kFull, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(kFull, l_run[r], 2);
        }
    }

    // This warp's state for the CTA's merge (after reduce_l): row h of the
    // accumulator at acc_rows[h * rs + d], each row's max and sum at m16[h]
    // and l16[h] (sum 0 when zero_l).
    __device__ __forceinline__ void store_merge(float* acc_rows, int rs, float* m16, float* l16,
                                                bool zero_l) const {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                float* base = acc_rows + (8 * r + 2 * cq) * rs + 16 * mt + gq;
                base[0] = acc[mt][r][0];
                base[rs] = acc[mt][r][1];
                base[8] = acc[mt][r][2];
                base[rs + 8] = acc[mt][r][3];
            }
        if (cq == 0) {
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                m16[8 * r + gq] = m_run[r];
                l16[8 * r + gq] = zero_l ? 0.f : l_run[r];
            }
        }
    }

    // This warp's state as a partial of each of its first `rows` rows:
    // o = acc / l times the output multiplier at ws_o[prow(h) * D + d], and
    // (max, sum) at ws_m / ws_l[prow(h)]; `dead` writes only an empty sum.
    template <class RowFn>
    __device__ __forceinline__ void write_partial(float* ws_o, float* ws_m, float* ws_l, int rows,
                                                  RowFn prow, bool dead) const {
#pragma unroll
        for (int hr = 0; hr < NH; ++hr) {
            float l = l_run[hr];
            l += __shfl_xor_sync(kFull, l, 1);
            l += __shfl_xor_sync(kFull, l, 2);
            const float lh[2] = {__shfl_sync(kFull, l, 8 * cq), __shfl_sync(kFull, l, 8 * cq + 4)};
            const float mh[2] = {__shfl_sync(kFull, m_run[hr], 8 * cq),
                                 __shfl_sync(kFull, m_run[hr], 8 * cq + 4)};
#pragma unroll
            for (int e1 = 0; e1 < 2; ++e1) {
                const int h = 8 * hr + 2 * cq + e1;
                if (h >= rows) continue;
                const long long pr = prow(h);
                const float L = dead ? 0.f : lh[e1];
                const float inv = L > 0.f ? out_mul / L : 0.f;
                if (!dead) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int e2 = 0; e2 < 2; ++e2)
                            ws_o[pr * D + 16 * mt + gq + 8 * e2] = acc[mt][hr][e1 + 2 * e2] * inv;
                }
                if (gq == 0) {
                    ws_m[pr] = mh[e1];
                    ws_l[pr] = L;
                }
            }
        }
    }

    // Fresh running state: max -inf, sum 0, accumulator 0.
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            m_run[r] = -INFINITY;
            l_run[r] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int r = 0; r < NH; ++r)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mt][r][e] = 0.f;
    }

    // One landed page: S = Q K^T, online softmax, O^T += V^T P^T.  FULL pages
    // (every slot a token) skip all masking.
    // `valid` (`valid2`): tokens of the stage's (second) page that count.
    template <bool FULL, bool ALIBI>
    __device__ __forceinline__ void page(const uint32_t kbase, const int valid, const int valid2,
                                         const int pos0) {
        const uint32_t vbase = kbase + NPG * PAGE;
        auto counts = [&](int tk) {  // token tk of the stage is part of the sequence
            if constexpr (PAIR) return tk < B ? tk < valid : tk - B < valid2;
            return tk < valid;
        };

        // ---------------- S = Q K^T  (rows: heads, cols: tokens)
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
        {
            const int mi = lane >> 3, r8 = lane & 7;
            if constexpr (!FP8) {
#pragma unroll
                for (int kt = 0; kt < KT; ++kt)
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        const int tok = 8 * (2 * np + (mi >> 1)) + r8;
                        const int chunk = 2 * kt + (mi & 1);
                        const uint32_t ka = PAIR ? kbase + np * PAGE + chunk * CHUNK +
                                                       (tok & 15) * 16
                                                 : kbase + chunk * CHUNK + tok * 16;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(ka, b0, b1, b2, b3);
                        mma_bf16_16816(sc[2 * np], qa[kt], b0, b1);
                        mma_bf16_16816(sc[2 * np + 1], qa[kt], b2, b3);
                    }
            } else if constexpr (F8MMA) {
                // K bytes go into the MMA as they are: register = 4 e4m3 codes of
                // d = 4 cq..4 cq+3 of a 16-d chunk of one token.
#pragma unroll
                for (int jp = 0; jp < K32; ++jp)
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        const int tok = 8 * (2 * np + (mi & 1)) + r8;
                        const int chunk = 2 * jp + (mi >> 1);
                        const uint32_t ka = PAIR ? kbase + np * PAGE + chunk * CHUNK +
                                                       (tok & 15) * 16
                                                 : kbase + chunk * CHUNK + tok * 16;
                        uint32_t w0, w1, w2, w3;
                        ldsm_x4(ka, w0, w1, w2, w3);
                        mma_e4m3_16832(sc[2 * np], qa8[jp][0], w0, w2);
                        mma_e4m3_16832(sc[2 * np], qa8[jp][1], w0, w2);
                        mma_e4m3_16832(sc[2 * np + 1], qa8[jp][0], w1, w3);
                        mma_e4m3_16832(sc[2 * np + 1], qa8[jp][1], w1, w3);
                    }
            } else {
#pragma unroll
                for (int jp = 0; jp < KT / 2; ++jp)
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        const int tok = 8 * (2 * np + (mi & 1)) + r8;
                        const int chunk = 2 * jp + (mi >> 1);
                        // With pairs, tokens 16 np .. 16 np + 15 are page np's.
                        const uint32_t ka = PAIR ? kbase + np * PAGE + chunk * CHUNK +
                                                       (tok & 15) * 16
                                                 : kbase + chunk * CHUNK + tok * 16;
                        uint32_t w0, w1, w2, w3;
                        ldsm_x4(ka, w0, w1, w2, w3);
                        const uint32_t(&qlo)[4] = qa[2 * jp];
                        const uint32_t(&qhi)[4] = qa[2 * jp + 1];
                        mma_f16_16816(sc[2 * np], qlo, e4m3_lo_pair(w0), e4m3_hi_pair(w0));
                        mma_f16_16816(sc[2 * np + 1], qlo, e4m3_lo_pair(w1), e4m3_hi_pair(w1));
                        mma_f16_16816(sc[2 * np], qhi, e4m3_lo_pair(w2), e4m3_hi_pair(w2));
                        mma_f16_16816(sc[2 * np + 1], qhi, e4m3_lo_pair(w3), e4m3_hi_pair(w3));
                    }
            }
        }

        // ---------------- online softmax (log2 domain), per head row
        uint32_t pp[NH][NT];
        float alpha[NH];
        bool grew = false;
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            float v[NT][2];
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float x = sc[nt][2 * r + e] * qk_mul;
                    if constexpr (ALIBI)
                        x = fmaf(slope2[r], static_cast<float>(pos0 + 8 * nt + 2 * cq + e), x);
                    if constexpr (!FULL) {
                        if (!counts(8 * nt + 2 * cq + e)) x = -INFINITY;
                    }
                    v[nt][e] = x;
                    mx = fmaxf(mx, x);
                }
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
            const float m_new = fmaxf(m_run[r], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            grew |= m_new > m_run[r];
            alpha[r] = fast_exp2(m_run[r] - m_use);
            m_run[r] = m_new;
            float ls = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float p0 = fast_exp2(v[nt][0] - m_use);
                const float p1 = fast_exp2(v[nt][1] - m_use);
                uint32_t w;
                if constexpr (F8MMA) {
                    // weights x 256 as hi + lo e4m3 codes (hi pair | lo pair << 16);
                    // the running sum uses the represented values, in the same x 256
                    // units as the accumulator.
                    float sum2;
                    w = split_e4m3x2(p0 * 256.f, p1 * 256.f, &sum2);
                    ls += sum2;
                } else if constexpr (!FP8) {
                    w = pack_bf16x2(p0, p1);
                    ls += bf16_lo(w) + bf16_hi(w);
                } else {
                    w = pack_f16x2(p0, p1);
                    ls += f16_lo(w) + f16_hi(w);
                }
                pp[r][nt] = w;
            }
            l_run[r] = l_run[r] * alpha[r] + ls;
        }

        // ---------------- rescale O^T columns (heads 8r + 2cq, 8r + 2cq + 1),
        // only when some row maximum of the warp moved.
        if (__any_sync(kFull, grew)) {
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                const float a0 = __shfl_sync(kFull, alpha[r], 8 * cq);
                const float a1 = __shfl_sync(kFull, alpha[r], 8 * cq + 4);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    acc[mt][r][0] *= a0;
                    acc[mt][r][1] *= a1;
                    acc[mt][r][2] *= a0;
                    acc[mt][r][3] *= a1;
                }
            }
        }

        if constexpr (F8MMA) {
            // O^T += V^T P^T with one 32-token e4m3 k-step per stage: tokens
            // 16 kk + 4 cq .. +3 of each k-tile come from the same quad shuffles
            // as below; V bytes go into the MMA as they are (with paired
            // 16-token pages, k-tile kk is page kk).
            uint32_t bh[NH][2], bl[NH][2];
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    if (kk < KK) {
                        const uint32_t x0 = __shfl_sync(kFull, pp[r][2 * kk], src0);
                        const uint32_t y0 = __shfl_sync(kFull, pp[r][2 * kk + 1], src0);
                        const uint32_t x1 = __shfl_sync(kFull, pp[r][2 * kk], src1);
                        const uint32_t y1 = __shfl_sync(kFull, pp[r][2 * kk + 1], src1);
                        const uint32_t u0 = hi_half ? y0 : x0;  // tokens 4cq, 4cq+1
                        const uint32_t u1 = hi_half ? y1 : x1;  // tokens 4cq+2, 4cq+3
                        bh[r][kk] = __byte_perm(u0, u1, 0x5410);
                        bl[r][kk] = __byte_perm(u0, u1, 0x7632);
                    } else {
                        bh[r][kk] = 0u;
                        bl[r][kk] = 0u;
                    }
                }
            uint32_t vmask[2] = {kFull, kFull};
            if constexpr (!FULL) {
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    const int t0 = 16 * kk + 4 * cq;
                    vmask[kk] = (counts(t0) ? 0x000000ffu : 0u) |
                                (counts(t0 + 1) ? 0x0000ff00u : 0u) |
                                (counts(t0 + 2) ? 0x00ff0000u : 0u) |
                                (counts(t0 + 3) ? 0xff000000u : 0u);
                }
            }
#pragma unroll
            for (int mp = 0; mp < MT / 2; ++mp) {
                uint32_t w[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    ldsm_x4(PAIR ? vbase + kk * PAGE + (32 * mp + lane) * B
                                 : vbase + (32 * mp + lane) * B + kk * 16,
                            w[kk][0], w[kk][1], w[kk][2], w[kk][3]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) w[kk][i] &= vmask[kk];
                }
                const uint32_t a0[4] = {w[0][0], w[0][1], w[1][0], w[1][1]};
                const uint32_t a1[4] = {w[0][2], w[0][3], w[1][2], w[1][3]};
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    mma_e4m3_16832(acc[2 * mp][r], a0, bh[r][0], bh[r][1]);
                    mma_e4m3_16832(acc[2 * mp][r], a0, bl[r][0], bl[r][1]);
                    mma_e4m3_16832(acc[2 * mp + 1][r], a1, bh[r][0], bh[r][1]);
                    mma_e4m3_16832(acc[2 * mp + 1][r], a1, bl[r][0], bl[r][1]);
                }
            }
        } else {
        // ---------------- O^T += V^T P^T  (rows: head dim, cols: heads, k: tokens)
        // Per 16-token k-tile, thread cq holds V for tokens 4cq..4cq+3 (one
        // contiguous 4-token group per row), so k = 2cq,2cq+1 <-> tokens
        // 4cq,4cq+1 and k = 2cq+8,2cq+9 <-> 4cq+2,4cq+3; P is regrouped to
        // that order with quad shuffles.
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            uint32_t pb0[NH], pb1[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                const uint32_t x0 = __shfl_sync(kFull, pp[r][2 * kk], src0);
                const uint32_t y0 = __shfl_sync(kFull, pp[r][2 * kk + 1], src0);
                const uint32_t x1 = __shfl_sync(kFull, pp[r][2 * kk], src1);
                const uint32_t y1 = __shfl_sync(kFull, pp[r][2 * kk + 1], src1);
                pb0[r] = hi_half ? y0 : x0;
                pb1[r] = hi_half ? y1 : x1;
            }
            // Slots past the sequence end may hold anything (even NaN); their
            // weights are 0, but 0 * NaN is NaN, so their V is zeroed.
            uint32_t mlo = kFull, mhi = kFull;
            if constexpr (!FULL) {
                const int t0 = 16 * kk + 4 * cq;
                mlo = (counts(t0) ? 0x0000ffffu : 0u) | (counts(t0 + 1) ? 0xffff0000u : 0u);
                mhi = (counts(t0 + 2) ? 0x0000ffffu : 0u) | (counts(t0 + 3) ? 0xffff0000u : 0u);
            }
            if constexpr (!FP8) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint32_t ra =
                        PAIR ? vbase + kk * PAGE + (16 * mt + gq) * (B * 2) + cq * 8
                             : vbase + (16 * mt + gq) * (B * 2) + kk * 32 + cq * 8;
                    const uint2 va = lds64(ra);
                    const uint2 vb = lds64(ra + 8 * (B * 2));
                    uint32_t a[4] = {va.x, vb.x, va.y, vb.y};
                    if constexpr (!FULL) {
                        a[0] &= mlo;
                        a[1] &= mlo;
                        a[2] &= mhi;
                        a[3] &= mhi;
                    }
#pragma unroll
                    for (int r = 0; r < NH; ++r) mma_bf16_16816(acc[mt][r], a, pb0[r], pb1[r]);
                }
            } else {
#pragma unroll
                for (int mp = 0; mp < MT / 2; ++mp) {
                    uint32_t w0, w1, w2, w3;
                    // With pairs, k-tile kk is page kk's 16 tokens.
                    ldsm_x4(PAIR ? vbase + kk * PAGE + (32 * mp + lane) * B
                                 : vbase + (32 * mp + lane) * B + kk * 16,
                            w0, w1, w2, w3);
                    uint32_t a0[4] = {e4m3_lo_pair(w0), e4m3_lo_pair(w1), e4m3_hi_pair(w0),
                                      e4m3_hi_pair(w1)};
                    uint32_t a1[4] = {e4m3_lo_pair(w2), e4m3_lo_pair(w3), e4m3_hi_pair(w2),
                                      e4m3_hi_pair(w3)};
                    if constexpr (!FULL) {
                        a0[0] &= mlo;
                        a0[1] &= mlo;
                        a0[2] &= mhi;
                        a0[3] &= mhi;
                        a1[0] &= mlo;
                        a1[1] &= mlo;
                        a1[2] &= mhi;
                        a1[3] &= mhi;
                    }
#pragma unroll
                    for (int r = 0; r < NH; ++r) {
                        mma_f16_16816(acc[2 * mp][r], a0, pb0[r], pb1[r]);
                        mma_f16_16816(acc[2 * mp + 1][r], a1, pb0[r], pb1[r]);
                    }
                }
            }
        }
        }  // e4m3 MMAs or f16/bf16 MMAs
    }
};

// One query head per kv head (MHA), bf16 pages: the same contract as
// WarpAttn, with q.K and P.V on the CUDA cores instead of tensor-core tiles
// whose 16 rows would hold one real head.  A stage holds BT = 16 or 32
// tokens (two 16-token pages of head size 64 are paired):
//   * q.K: lane l takes head dims [part DL, (part + 1) DL), part = l / 8,
//     DL = D / 4, and tokens l % 8 + 8 j, reading each token's 16-byte
//     column groups of the K page (8 consecutive head dims); the 8 lanes of
//     a shared-memory phase read 8 different tokens, so 8 different banks.
//     Two xor shuffles add the four parts;
//   * softmax in fp32 over the stage's tokens with xor shuffles;
//   * P.V: the weights go through the first bytes of the stage's (already
//     read) K page and come back as broadcast float4 loads; lane l owns head
//     dims l + 32 i and reads its V rows' 16-byte pieces in an order that
//     keeps the 8 lanes of a phase on distinct banks.
// The weights stay fp32 (not rounded to bf16 as the MMA operands are).
template <int D, int B>
struct WarpAttnScalar {
    static constexpr bool PAIR = pair_pages<D, B, false, false>();
    static constexpr int NPG = PAIR ? 2 : 1;  // logical pages per stage
    static constexpr int BT = B * NPG;        // tokens per stage
    static constexpr int PAGE = D * B * 2;    // one bf16 K (or V) page of one kv head
    static constexpr int CHUNK = B * 16;      // bytes of one 16-byte column group of a K page
    static constexpr int DL = D / 4;          // head dims per lane in q.K
    static constexpr int TJ = BT / 8;         // tokens per lane in q.K
    static constexpr int DV = D / 32;         // head dims per lane in P.V

    int lane, tl, part;
    uint4 qw[DL / 8];  // raw query words until finish_query
    float q[DL];
    float qk_mul, out_mul;
    float slope2[1];
    float m_run[1], l_run[1];
    float acc[DV];

    __device__ __forceinline__ explicit WarpAttnScalar(int lane_) {
        lane = lane_;
        tl = lane & 7;
        part = lane >> 3;
    }

    template <class RowFn>
    __device__ __forceinline__ void fetch_query(const uint16_t* qp, RowFn row_of) {
        const long long qr = row_of(0);
        const uint4* src = reinterpret_cast<const uint4*>(qp + (qr >= 0 ? qr : 0) * D + part * DL);
#pragma unroll
        for (int c = 0; c < DL / 8; ++c) qw[c] = qr >= 0 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }

    __device__ __forceinline__ void finish_query(float scale_log2, float, float) {
#pragma unroll
        for (int c = 0; c < DL / 8; ++c) {
            const uint32_t w[4] = {qw[c].x, qw[c].y, qw[c].z, qw[c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                q[8 * c + 2 * k] = bf16_lo(w[k]);
                q[8 * c + 2 * k + 1] = bf16_hi(w[k]);
            }
        }
        qk_mul = scale_log2;
        out_mul = 1.f;
    }

    template <class RowFn>
    __device__ __forceinline__ void set_alibi(const float* alibi, int Hq, RowFn row_of) {
        const long long qr = row_of(0);
        slope2[0] = (alibi && qr >= 0) ? __ldg(alibi + qr % Hq) * 1.4426950408889634f : 0.f;
    }

    __device__ __forceinline__ void reset() {
        m_run[0] = -INFINITY;
        l_run[0] = 0.f;
#pragma unroll
        for (int i = 0; i < DV; ++i) acc[i] = 0.f;
    }

    // Every lane holds the row's sum already.
    __device__ __forceinline__ void reduce_l() {}

    __device__ __forceinline__ void store_merge(float* acc_rows, int, float* m16, float* l16,
                                                bool zero_l) const {
#pragma unroll
        for (int i = 0; i < DV; ++i) acc_rows[lane + 32 * i] = acc[i];
        if (lane == 0) {
            m16[0] = m_run[0];
            l16[0] = zero_l ? 0.f : l_run[0];
        }
    }

    template <class RowFn>
    __device__ __forceinline__ void write_partial(float* ws_o, float* ws_m, float* ws_l, int rows,
                                                  RowFn prow, bool dead) const {
        if (rows < 1) return;
        const long long pr = prow(0);
        const float L = dead ? 0.f : l_run[0];
        const float inv = L > 0.f ? out_mul / L : 0.f;
        if (!dead) {
#pragma unroll
            for (int i = 0; i < DV; ++i) ws_o[pr * D + lane + 32 * i] = acc[i] * inv;
        }
        if (lane == 0) {
            ws_m[pr] = m_run[0];
            ws_l[pr] = L;
        }
    }

    template <bool FULL, bool ALIBI>
    __device__ __forceinline__ void page(const uint32_t kbase, const int valid, const int valid2,
                                         const int pos0) {
        const uint32_t vbase = kbase + NPG * PAGE;
        // ---------------- logits of tokens tl + 8 j (this lane's quarter of the head dims)
        float x[TJ];
#pragma unroll
        for (int j = 0; j < TJ; ++j) {
            const int tok = tl + 8 * j;
            const int pg = PAIR ? tok / B : 0;
            const uint32_t kp = kbase + pg * PAGE + (tok % B) * 16 + part * (DL / 8) * CHUNK;
            float sc = 0.f;
#pragma unroll
            for (int c = 0; c < DL / 8; ++c) {
                const uint4 w = lds128(kp + c * CHUNK);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sc = fmaf(q[8 * c + 2 * k], bf16_lo(ww[k]), sc);
                    sc = fmaf(q[8 * c + 2 * k + 1], bf16_hi(ww[k]), sc);
                }
            }
            sc += __shfl_xor_sync(kFull, sc, 8);
            sc += __shfl_xor_sync(kFull, sc, 16);
            float v = sc * qk_mul;
            if constexpr (ALIBI) v = fmaf(slope2[0], static_cast<float>(pos0 + tok), v);
            if constexpr (!FULL) {
                const bool counts = PAIR ? (tok < B ? tok < valid : tok - B < valid2) : tok < valid;
                if (!counts) v = -INFINITY;
            }
            x[j] = v;
        }
        // ---------------- online softmax over the stage's tokens
        float mx = x[0];
#pragma unroll
        for (int j = 1; j < TJ; ++j) mx = fmaxf(mx, x[j]);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        const float m_new = fmaxf(m_run[0], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const bool grew = m_new > m_run[0];
        const float alpha = fast_exp2(m_run[0] - m_use);
        m_run[0] = m_new;
        float pw[TJ];
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < TJ; ++j) {
            pw[j] = fast_exp2(x[j] - m_use);
            ls += pw[j];
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) ls += __shfl_xor_sync(kFull, ls, o);
        l_run[0] = l_run[0] * alpha + ls;
        if (grew) {
#pragma unroll
            for (int i = 0; i < DV; ++i) acc[i] *= alpha;
        }
        // ---------------- weights to every lane through the stage's K page
        __syncwarp();  // every lane has read its K words
        if (part == 0) {
#pragma unroll
            for (int j = 0; j < TJ; ++j) sts32(kbase + 4 * (tl + 8 * j), __float_as_uint(pw[j]));
        }
        __syncwarp();
        float pv[BT];
#pragma unroll
        for (int c = 0; c < BT / 4; ++c) {
            const uint4 w = lds128(kbase + 16 * c);
            pv[4 * c] = __uint_as_float(w.x);
            pv[4 * c + 1] = __uint_as_float(w.y);
            pv[4 * c + 2] = __uint_as_float(w.z);
            pv[4 * c + 3] = __uint_as_float(w.w);
        }
        // ---------------- O += V P for head dims lane + 32 i
        // A V row of one page is PIECES 16-byte pieces of 8 tokens.  Lanes of
        // one 8-lane shared-memory phase start on different pieces (rot), so
        // their loads land on distinct banks; the piece index is then a
        // run-time value, and each weight is picked from the pieces' weights.
        constexpr int PIECES = B * 2 / 16;
        const int rot = PIECES == 2 ? (lane >> 2) & 1 : (lane >> 1) & 3;
#pragma unroll
        for (int pgv = 0; pgv < NPG; ++pgv) {
            const int cnt = FULL ? B : (pgv == 0 ? valid : valid2);
#pragma unroll
            for (int i = 0; i < DV; ++i) {
                const uint32_t row = vbase + pgv * PAGE + (lane + 32 * i) * (B * 2);
#pragma unroll
                for (int hh = 0; hh < PIECES; ++hh) {
                    const int h = (hh + rot) % PIECES;
                    const uint4 w = lds128(row + 16 * h);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float pj = pv[pgv * B + j];
#pragma unroll
                        for (int hc = 1; hc < PIECES; ++hc)
                            pj = (h == hc) ? pv[pgv * B + 8 * hc + j] : pj;
                        float v = (j & 1) ? bf16_hi(ww[j >> 1]) : bf16_lo(ww[j >> 1]);
                        if constexpr (!FULL) v = 8 * h + j < cnt ? v : 0.f;  // slots past the end may hold NaN
                        acc[i] = fmaf(pj, v, acc[i]);
                    }
                }
            }
        }
    }
};

// What a row's merge needs once its slots' loads are in flight: how many
// slots it has (< 0: nothing to do, the decode kernel wrote the row) and
// which row of out it writes.
struct SlotRow {
    int nps;
    long long out_row;
};

// The merge of one row whose slots fit in a warp (at most 32), at partial
// rows base .. base + np - 1: every load it needs -- each slot's (max, sum),
// one slot per lane, the partial rows of the first 16 slots (D / 32
// consecutive head dims per lane), and whatever row_info reads -- is issued
// before any of them is used, so a row costs one memory round trip (a second
// one for slots 16..31).  Slots past the row's count (and an empty slot's
// row) may hold anything; their weight is 0 and a select drops them.  The
// partials are read through L2 (other CTAs of the same kernel may have just
// written them).
template <int D, class RowInfo>
__device__ __forceinline__ void merge_slots(const float* ws_o, const float* ws_m,
                                            const float* ws_l, __nv_bfloat16* out,
                                            long long base, int np, int lane, RowInfo row_info) {
    constexpr int V = D / 32;  // head dims per lane: 4 * lane .. (D = 128) or 2 * lane ..
    constexpr int KO = 16;     // partial rows loaded up front
    float l = 0.f, m = -INFINITY;
    if (lane < np) {
        l = __ldcg(ws_l + base + lane);
        m = __ldcg(ws_m + base + lane);
    }
    auto load_row = [&](int i, float (&v)[V]) {
        const float* src = ws_o + (base + i) * D + V * lane;
        if constexpr (V == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(src));
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        } else {
            const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
            v[0] = x.x; v[1] = x.y;
        }
    };
    float o[KO][V];
#pragma unroll
    for (int i = 0; i < KO; ++i) {
        if (i < np) {
            load_row(i, o[i]);
        } else {
#pragma unroll
            for (int j = 0; j < V; ++j) o[i][j] = 0.f;
        }
    }
    const SlotRow r = row_info();
    if (r.nps < 0) return;
    const int nps = r.nps;
    const bool live = lane < nps && l > 0.f;
    float M = live ? m : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
    const float wt = live ? exp2f(m - M) * l : 0.f;
    float L = wt;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(kFull, L, off);
    float a[V];
#pragma unroll
    for (int j = 0; j < V; ++j) a[j] = 0.f;
#pragma unroll
    for (int i = 0; i < KO; ++i) {
        const float w = __shfl_sync(kFull, wt, i);
#pragma unroll
        for (int j = 0; j < V; ++j) a[j] += w > 0.f ? w * o[i][j] : 0.f;
    }
    for (int i0 = KO; i0 < nps; i0 += 8) {
        float q[8][V];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i0 + i < nps) {
                load_row(i0 + i, q[i]);
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j) q[i][j] = 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float w = __shfl_sync(kFull, wt, (i0 + i) & 31);
#pragma unroll
            for (int j = 0; j < V; ++j) a[j] += (i0 + i < nps && w > 0.f) ? w * q[i][j] : 0.f;
        }
    }
    __nv_bfloat16* dst = out + r.out_row * D + V * lane;
#pragma unroll
    for (int j = 0; j < V; j += 2) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(L > 0.f ? a[j] / L : 0.f,
                                                       L > 0.f ? a[j + 1] / L : 0.f);
        *reinterpret_cast<__nv_bfloat162*>(dst + j) = h;
    }
}

// Shared-prefix units: a CTA streams one partition of one kv head's prefix
// pages once, through one ring of W * stages page buffers shared by its W
// warps, and warp w keeps the running state of 16-row group cg * W + w of
// that kv head's query rows -- so the pages are read once for W groups
// instead of once per group.  Warp 0 issues every page's copies; a buffer is
// refilled once every active warp has released it (an "empty" mbarrier with
// one arrival per active warp, beside the "full" one the copies complete),
// and a word per buffer tells the warps which of its pages had a legal block
// id (written before the "full" arrival, so its completion publishes it).
// Each warp then writes its rows' partials (slot `part`) itself.  Every wait
// is bounded; one that gives up stops the warp, and warp 0 lets the copies it
// issued land before the CTA can exit.
template <class WS, int D, int B, bool FP8, bool PAIR, int W>
__device__ __forceinline__ void prefix_shared_ring(const DecodeParams& p, uint32_t sbase,
                                                   uint32_t bars, int kvh, int cg, int part) {
    constexpr int PAGE = D * B * (FP8 ? 1 : 2);
    constexpr int NPG = PAIR ? 2 : 1;
    constexpr int STAGE = 2 * PAGE * NPG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nsh = W * p.stages;  // shared page buffers
    const uint32_t full0 = bars, empty0 = bars + 8 * nsh, flags0 = bars + 16 * nsh;
    const int n_active = min(W, p.prefix_groups - cg * W);
    if (threadIdx.x == 0) {
        for (int i = 0; i < nsh; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, n_active);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int rg = cg * W + warp;
    if (rg >= p.prefix_groups) return;  // no group for this warp (issues nothing)

    const int j0 = part * p.PP;
    const int j1 = min(p.prefix_pages, j0 + p.PP);
    const int span = (j1 - j0 + NPG - 1) / NPG;  // stages of this partition
    const int rows_total = p.S * p.G;
    auto row_of = [&](int lr) -> long long {
        const int gi = rg * 16 + lr;
        if (gi >= rows_total) return -1;
        return (long long)(gi / p.G) * p.Hq + (long long)kvh * p.G + gi % p.G;
    };
    // Warp 0's block-table window: lane l holds stage (wbase + l)'s page.
    const int32_t* btrow = p.bt;  // the prefix is row 0's first blocks
    auto load_win = [&](int base, int off) -> int {
        const int j = j0 + NPG * (base + lane) + off;
        return j < j1 ? __ldg(btrow + j) : -1;
    };
    int win_a = -1, win_b = -1, win_a2 = -1, win_b2 = -1, wbase = 0;
    if (warp == 0) {
        win_a = load_win(0, 0);
        win_b = load_win(32, 0);
        if constexpr (PAIR) {
            win_a2 = load_win(0, 1);
            win_b2 = load_win(32, 1);
        }
    }
    WS wa(lane);
    wa.fetch_query(p.q, row_of);
    float k_scale = 1.f, v_scale = 1.f;
    if constexpr (FP8) {
        k_scale = __ldg(p.k_scale);
        v_scale = __ldg(p.v_scale);
    }
    wa.set_alibi(nullptr, p.Hq, row_of);
    const size_t head_off = static_cast<size_t>(kvh) * PAGE;
    const size_t block_stride = static_cast<size_t>(p.Hk) * PAGE;
    // Copies of stage i (warp 0 only, stages in increasing order).
    auto issue = [&](int i) {
        if (i >= wbase + 32) {
            win_a = win_b;
            win_b = load_win(wbase + 64, 0);
            if constexpr (PAIR) {
                win_a2 = win_b2;
                win_b2 = load_win(wbase + 64, 1);
            }
            wbase += 32;
        }
        const int pb = __shfl_sync(kFull, win_a, i & 31);
        const int pb2 = PAIR ? __shfl_sync(kFull, win_a2, i & 31) : -1;
        const int st = i % nsh;
        const uint32_t bar = full0 + 8 * st;
        const bool ok = pb >= 0 && static_cast<long long>(pb) < p.num_blocks;
        const bool has2 = PAIR && j0 + NPG * i + 1 < j1;
        const bool ok2 = has2 && pb2 >= 0 && static_cast<long long>(pb2) < p.num_blocks;
        if (lane == 0) {
            sts32(flags0 + 4 * st, (ok ? 1u : 0u) | (ok2 ? 2u : 0u));
            const uint32_t bytes = (ok ? 2 * PAGE : 0) + (ok2 ? 2 * PAGE : 0);
            const uint32_t dst = sbase + static_cast<uint32_t>(st * STAGE);
            if (bytes) {
                mbar_arrive_expect_tx(bar, bytes + p.stall_tx_bytes);
                if (ok) {
                    const size_t off = static_cast<size_t>(pb) * block_stride + head_off;
                    bulk_copy_g2s(dst, p.kc + off, PAGE, bar);
                    bulk_copy_g2s(dst + NPG * PAGE, p.vc + off, PAGE, bar);
                }
                if (ok2) {
                    const size_t off = static_cast<size_t>(pb2) * block_stride + head_off;
                    bulk_copy_g2s(dst + PAGE, p.kc + off, PAGE, bar);
                    bulk_copy_g2s(dst + 3 * PAGE, p.vc + off, PAGE, bar);
                }
            } else {
                mbar_arrive(bar);
            }
            if (!ok || (has2 && !ok2)) atomicOr(p.status, kDevBadBlock);
        }
    };
    int issued = 0;
    if (warp == 0) {
        for (; issued < min(span, nsh); ++issued) issue(issued);
    }
    wa.finish_query(p.scale_log2, k_scale, v_scale);
    wa.reset();

    bool timed_out = false;
    int k = 0;
    for (; k < span; ++k) {
        const int st = k % nsh;
        const uint32_t ph = static_cast<uint32_t>(k / nsh) & 1u;
        if (!__all_sync(kFull, mbar_wait_bounded(full0 + 8 * st, ph, p.wait_limit_ns))) {
            timed_out = true;
            break;
        }
        // Prefix pages are whole blocks: every slot of a legal page is a token
        // (a stage past the partition's last pair holds one page).
        const uint32_t fl = lds32(flags0 + 4 * st);
        const int valid = (fl & 1u) ? B : 0;
        const int valid2 = (fl & 2u) ? B : 0;
        const uint32_t kb = sbase + static_cast<uint32_t>(st * STAGE);
        if (valid == B && (!PAIR || valid2 == B))
            wa.template page<true, false>(kb, B, B, 0);
        else
            wa.template page<false, false>(kb, valid, valid2, 0);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * st);
        if (warp == 0 && issued < span) {
            // Buffer st is free once every active warp has released stage k.
            if (!__all_sync(kFull, mbar_wait_bounded(empty0 + 8 * st, ph, p.wait_limit_ns))) {
                timed_out = true;
                ++k;  // stage k was consumed
                break;
            }
            issue(issued++);
        }
    }
    if (timed_out) {
        if (warp == 0) {
            // Let every copy issued and not yet seen land (bounded) before the
            // CTA's shared memory can be handed to anyone else.
            for (int i = k; i < issued; ++i)
                (void)mbar_wait_bounded(full0 + 8 * (i % nsh),
                                        static_cast<uint32_t>(i / nsh) & 1u, p.wait_limit_ns);
        }
        if (lane == 0) atomicOr(p.status, kDevTimeout);
    }
    const int rows_here = min(16, rows_total - rg * 16);
    wa.write_partial(p.ws_o, p.ws_m, p.ws_l, rows_here,
                     [&](int h) { return row_of(h) * p.P_total + part; }, timed_out);
}

// The paired 8-row form with f16 MMAs is held to three CTAs per SM (170
// registers), the residency of the other 8-row forms.
// SC: one query head per kv head on the CUDA cores (WarpAttnScalar).
template <int D, int B, bool FP8, int NH, int W, bool F8MMA, bool SC = false>
__global__ void __launch_bounds__(W * 32,
                                  ((pair_pages<D, B, FP8, F8MMA>() && !F8MMA && NH == 1) || SC) ? 3
                                                                                                : 1)
    pa_decode_kernel(const DecodeParams p) {
    static_assert(!F8MMA || FP8, "e4m3 MMAs need e4m3 pages");
    static_assert(!SC || (!FP8 && NH == 1), "the CUDA-core form takes bf16 pages and one head");
    using WA = std::conditional_t<SC, WarpAttnScalar<D, B>, WarpAttn<D, B, FP8, NH, F8MMA>>;
    constexpr int ELEM = FP8 ? 1 : 2;
    constexpr int PAGE = D * B * ELEM;  // one K (or V) page of one kv head
    // Small pages go in pairs (pair_pages): a stage holds two
    // consecutive logical blocks of the unit (K a, K b, V a, V b), so a warp
    // keeps as many bytes in flight as with 32-token pages, and one pass of
    // the page code covers 32 tokens.
    constexpr bool PAIR = pair_pages<D, B, FP8, F8MMA>();
    constexpr int NPG = PAIR ? 2 : 1;  // logical pages per stage
    constexpr int STAGE = 2 * PAGE * NPG;
    constexpr int RS = D + 4;      // padded row stride of the merge buffer

    extern __shared__ __align__(128) uint8_t smem[];

    // Launched with programmatic stream serialization: wait for the kernel
    // ahead in the stream (which may write the inputs) before any access, and
    // let the next kernel (the combine, or the next call) be scheduled now;
    // it waits for this grid to complete in turn.
    grid_dep_wait();
    grid_dep_launch_dependents();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---------------- this CTA's work: one unit, or a balanced page range
    bool pre = false;  // a shared-prefix unit
    int kvh = 0, s = 0, part = 0, rg = 0;
    long long tail_t = -1;  // unit of the split tail, or -1
    long long bx = 0, bx_first = 0, bx_end = 0;  // balanced: pages [bx, bx_end) still to do
    int bj = 0, bn = 0;                          // balanced: page in the unit, pages of the unit
    const int t_cap = p.max_blocks * B;
    auto pages_of = [&](int seq) {
        const int t = max(0, min(__ldg(p.seq_lens + seq), t_cap));
        return (t + B - 1) / B;
    };
    if (p.balanced) {
        // Pages of every sequence and their exclusive prefix sum, at the start
        // of shared memory (no page is in flight yet): scan[i] for i < S, the
        // total at scan[S], then one partial sum per thread.
        int* scan = reinterpret_cast<int*>(smem);
        int* tsum = scan + p.S + 1;
        constexpr int NT = W * 32;
        const int chunk = (p.S + NT - 1) / NT;
        const int i0 = min(p.S, static_cast<int>(threadIdx.x) * chunk);
        const int i1 = min(p.S, i0 + chunk);
        int local = 0;
        bool bad_len = false;
        for (int i = i0; i < i1; ++i) {
            const int t = __ldg(p.seq_lens + i);
            bad_len |= t < 0 || t > t_cap;
            const int n = pages_of(i);
            scan[i] = n;
            local += n;
        }
        if (bad_len && blockIdx.x == 0) atomicOr(p.status, kDevSeqLen);
        tsum[threadIdx.x] = local;
        __syncthreads();
        if (threadIdx.x == 0) {
            int run = 0;
            for (int t = 0; t < NT; ++t) {
                const int v = tsum[t];
                tsum[t] = run;
                run += v;
            }
            scan[p.S] = run;
        }
        __syncthreads();
        int run = tsum[threadIdx.x];
        for (int i = i0; i < i1; ++i) {
            const int v = scan[i];
            scan[i] = run;
            run += v;
        }
        __syncthreads();
        const long long total = static_cast<long long>(p.Hk) * scan[p.S];
        const long long per = max(1LL, (total + gridDim.x - 1) / gridDim.x);
        bx = static_cast<long long>(blockIdx.x) * per;
        bx_first = bx;
        bx_end = min(total, bx + per);
        if (blockIdx.x == 0) {
            for (int i = threadIdx.x; i <= p.S; i += NT) p.br_scan[i] = scan[i];
            if (threadIdx.x == 0) p.br_scan[p.S + 1] = static_cast<int>(per);
        }
        if (bx < bx_end) {
            // The sequence holding page bx: the largest s with Hk scan[s] <= bx.
            // It has pages, since bx < Hk scan[S].
            int lo = 0, hi = p.S - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (static_cast<long long>(p.Hk) * scan[mid] <= bx)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            s = lo;
            bn = scan[s + 1] - scan[s];
            const long long off = bx - static_cast<long long>(p.Hk) * scan[s];
            kvh = static_cast<int>(off / bn);
            bj = static_cast<int>(off - static_cast<long long>(kvh) * bn);
        }
        __syncthreads();  // the scratch is page memory from here on
        if (bx >= bx_end) return;  // no work for this CTA (same for all its threads)
    } else {
        const long long unit = blockIdx.x;
        pre = unit < p.prefix_units;
        if (pre) {
            kvh = static_cast<int>(unit % p.Hk);
            // the row group (or, shared, the group of W row groups)
            rg = static_cast<int>((unit / p.Hk) % p.prefix_cta_groups);
            part = static_cast<int>(unit / ((long long)p.Hk * p.prefix_cta_groups));
            s = 0;
        } else {
            long long u = unit - p.prefix_units;
            if (p.tail_P > 0 && u >= p.n_full) {
                // A partition of a split-tail unit (all of them follow the
                // whole units, partition-major).
                const long long n_tail = static_cast<long long>(p.Hk) * p.S - p.n_full;
                const long long t = u - p.n_full;
                tail_t = t % n_tail;
                part = static_cast<int>(t / n_tail);
                u = p.n_full + tail_t;
            } else {
                part = static_cast<int>(u / ((long long)p.Hk * p.S));
            }
            kvh = static_cast<int>(u % p.Hk);
            s = static_cast<int>((u / p.Hk) % p.S);
            if (p.longest_first) {
                // The unit's sequence index is a rank: find the sequence with
                // that rank among all lengths, longest first, so that the
                // longest work starts first and the last wave of CTAs is short.
                // Uses the start of shared memory, which holds no page yet.
                int* lens = reinterpret_cast<int*>(smem);
                const int len0 = max(0, min(__ldg(p.seq_lens), t_cap));
                int differs = 0;
                for (int i = threadIdx.x; i < p.S; i += W * 32) {
                    lens[i] = max(0, min(__ldg(p.seq_lens + i), t_cap));
                    differs |= lens[i] != len0;
                }
                // Equal lengths (a block-wide vote): index order is already
                // longest first.  Otherwise every sequence's rank is counted and
                // the one whose rank is the unit's index is picked.
                if (__syncthreads_or(differs)) {
                    for (int i = threadIdx.x; i < p.S; i += W * 32) {
                        const int v = lens[i];
                        int rank = 0;
                        for (int j = 0; j < p.S; ++j) {
                            const int w2 = lens[j];
                            rank += (w2 > v) | ((w2 == v) & (j < i));
                        }
                        if (rank == s) lens[p.S] = i;
                    }
                    __syncthreads();
                    s = lens[p.S];
                }
                __syncthreads();  // the scratch is page memory from here on
            }
        }
    }

    // Shared memory: per-warp page stages, then the mbarriers.  The ring keeps
    // its stage / phase counters across a CTA's segments (every segment
    // consumes all it issued).
    const int NS = p.stages;
    const uint32_t sbase = smem_addr(smem);
    if constexpr (NH == 2 && !SC) {
        if (pre && p.prefix_shared) {  // (barriers, page flags after the stage area)
            const int area = max(W * NS * STAGE, merge_smem_bytes<D, NH, W>());
            prefix_shared_ring<WA, D, B, FP8, PAIR, W>(p, sbase, sbase + area, kvh, rg, part);
            return;
        }
    }
    const uint32_t wstage0 = sbase + static_cast<uint32_t>(warp * NS * STAGE);
    // mbarriers sit after the larger of the page stages and the merge buffer
    // that later overlays them (the host sizes shared memory the same way).
    const int stage_area = max(W * NS * STAGE, merge_smem_bytes<D, NH, W>());
    const uint32_t bar0 = sbase + static_cast<uint32_t>(stage_area + warp * NS * 8);
    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
    }
    __syncwarp();
    int stage = 0;
    uint32_t phase = 0;
    int issue_stage = 0;

    for (;;) {  // one segment per pass (a single pass unless balanced)
        const bool cascade = p.prefix_pages > 0;
        const int pg0 = pre ? 0 : p.prefix_pages;  // first page of this unit's page range
        const int PPu = tail_t >= 0 ? p.tail_PP : p.PP;  // the unit's partition size and count
        const int Pu = tail_t >= 0 ? p.tail_P : p.P;
        const int j0 = p.balanced ? bj : pg0 + part * PPu;
        const long long row0 = (long long)s * p.Hq + (long long)kvh * p.G;  // first q head row
        const int rows_total = p.S * p.G;  // query rows of one kv head (prefix units)

        // Query row (s*Hq + head) of local row lr = 8r + gq, or -1 when unused.
        auto row_of = [&](int lr) -> long long {
            if (pre) {
                const int gi = rg * 16 + lr;
                if (gi >= rows_total) return -1;
                return (long long)(gi / p.G) * p.Hq + (long long)kvh * p.G + gi % p.G;
            }
            return lr < p.G ? row0 + lr : -1;
        };

        // Loads that do not depend on the sequence length go out first, so their
        // latencies overlap: the block-table window (every entry of the row up to
        // the partition's end is readable), the raw query words and the scales.
        // Block-table window: lane l holds the id of this warp's page (wbase + l).
        const int32_t* btrow = p.bt + (long long)s * p.max_blocks;
        const int jcap = p.balanced ? min(bn, p.max_blocks)
                                    : min(j0 + PPu, pre ? p.prefix_pages : p.max_blocks);
        // (A stage's first page; with pairs, `off` = 1 reads its second.)
        auto load_win = [&](int base, int off) -> int {
            const int j = j0 + NPG * (warp + W * (base + lane)) + off;
            return j < jcap ? __ldg(btrow + j) : -1;
        };
        int win_a = load_win(0, 0);
        int win_b = load_win(32, 0);
        int win_a2 = PAIR ? load_win(0, 1) : -1;
        int win_b2 = PAIR ? load_win(32, 1) : -1;
        // The query rows, as MMA operands (or CUDA-core registers) later.
        WA wa(lane);
        wa.fetch_query(p.q, row_of);
        float k_scale = 1.f, v_scale = 1.f;
        if constexpr (FP8) {
            k_scale = __ldg(p.k_scale);
            v_scale = __ldg(p.v_scale);
        }
        const bool has_alibi = p.alibi != nullptr;
        wa.set_alibi(p.alibi, p.Hq, row_of);

        // ---- sequence length, with the device-side range checks
        int T, nb;
        if (pre) {
            nb = p.prefix_pages;  // every prefix page is full
            T = nb * B;
        } else {
            T = __ldg(p.seq_lens + s);
            uint32_t bad = 0;
            if (T < 0) { T = 0; bad = kDevSeqLen; }
            if (T > t_cap) { T = t_cap; bad = kDevSeqLen; }
            nb = (T + B - 1) / B;
            const int covered = p.balanced ? nb : pg0 + Pu * PPu;
            if (nb > covered) { nb = covered; T = nb * B; bad = kDevSeqLen; }
            if (cascade && T < p.prefix_pages * B) bad |= kDevPrefix;
            if (bad && part == 0 && kvh == 0 && j0 == pg0 && threadIdx.x == 0)
                atomicOr(p.status, bad);
            if (cascade && part == 0 && kvh == 0 && warp == 0 && s > 0) {
                // The declared prefix must be the same physical blocks as row 0's.
                bool same = true;
                for (int j = lane; j < p.prefix_pages; j += 32)
                    same &= __ldg(btrow + j) == __ldg(p.bt + j);
                if (!__all_sync(kFull, same) && lane == 0) atomicOr(p.status, kDevPrefix);
            }
        }

        // Balanced: the segment ends with the unit or with the CTA's range.
        const int j1 = p.balanced
                           ? static_cast<int>(min(static_cast<long long>(nb), j0 + (bx_end - bx)))
                           : min(nb, j0 + PPu);
        const bool direct = !cascade && (p.balanced ? (j0 == 0 && j1 == nb)
                                                    : ((Pu == 1) || (nb <= PPu)));

        // Split tail: once this CTA's partial rows are stored (or it had no
        // pages), it counts itself in on its unit; the unit's last CTA merges
        // the partials of its partitions that have pages (a warp per row, as
        // pa_combine_kernel does) into out -- unless one partition held the
        // whole sequence and wrote out itself -- and leaves the count at 0.
        auto tail_arrive = [&]() {
            __threadfence();  // this thread's partial stores before the count
            __syncthreads();
            int last = 0;
            if (threadIdx.x == 0)
                last = atomicAdd(p.merge_cnt + tail_t, 1u) == static_cast<unsigned>(p.tail_P - 1);
            if (!__syncthreads_or(last)) return;
            __threadfence();  // the other partitions' partials before reading them
            if (threadIdx.x == 0) p.merge_cnt[tail_t] = 0u;  // all of the unit's CTAs are in
            const int nps = min(p.tail_P, (nb + p.tail_PP - 1) / p.tail_PP);
            if (nps <= 1) return;
            const long long prow0 = tail_t * p.G * p.tail_P;
            for (int g = warp; g < p.G; g += W)
                merge_slots<D>(p.ws_o, p.ws_m, p.ws_l, p.out, prow0 + g * p.tail_P, p.tail_P,
                               lane, [&]() -> SlotRow { return {nps, row0 + g}; });
        };

        if (j0 >= j1) {
            if (!cascade && part == 0) {  // empty sequence: defined as a zero output row
                for (int i = threadIdx.x; i < p.G * D; i += (W * 32))
                    p.out[row0 * D + i] = __float2bfloat16_rn(0.f);
            }
            if (tail_t >= 0) tail_arrive();
            return;
        }

        const int span = (j1 - j0 + NPG - 1) / NPG;  // stages of this segment
        const int n_my = span > warp ? (span - warp + W - 1) / W : 0;

        int wbase = 0;
        // Bit NPG * stage (+ 1): the stage's (second) page had a legal block id.
        uint32_t valid_mask = 0;

        const size_t head_off = static_cast<size_t>(kvh) * PAGE;
        const size_t block_stride = static_cast<size_t>(p.Hk) * PAGE;

        // Issue the copies of this warp's i-th page (warp-uniform call, pages in
        // increasing order).  Pages go to consecutive stages of the ring, starting
        // where the consumer stands; `issue_stage` tracks that without a division.
        issue_stage = stage;
        auto issue = [&](int i) {
            if (i >= wbase + 32) {
                win_a = win_b;
                win_b = load_win(wbase + 64, 0);
                if constexpr (PAIR) {
                    win_a2 = win_b2;
                    win_b2 = load_win(wbase + 64, 1);
                }
                wbase += 32;
            }
            const int pb = __shfl_sync(kFull, win_a, i & 31);
            const int pb2 = PAIR ? __shfl_sync(kFull, win_a2, i & 31) : -1;
            const int stage = issue_stage;
            issue_stage = (issue_stage + 1 == NS) ? 0 : issue_stage + 1;
            const uint32_t bar = bar0 + 8 * stage;
            const bool ok = pb >= 0 && static_cast<long long>(pb) < p.num_blocks;
            // With pairs, the second page belongs to the stage only inside the segment.
            const bool has2 = PAIR && j0 + NPG * (warp + W * i) + 1 < j1;
            const bool ok2 = has2 && pb2 >= 0 && static_cast<long long>(pb2) < p.num_blocks;
            if (lane == 0) {
                const uint32_t bytes = (ok ? 2 * PAGE : 0) + (ok2 ? 2 * PAGE : 0);
                const uint32_t dst = wstage0 + static_cast<uint32_t>(stage * STAGE);
                if (bytes) {
                    mbar_arrive_expect_tx(bar, bytes + p.stall_tx_bytes);
                    if (ok) {
                        const size_t off = static_cast<size_t>(pb) * block_stride + head_off;
                        bulk_copy_g2s(dst, p.kc + off, PAGE, bar);
                        bulk_copy_g2s(dst + NPG * PAGE, p.vc + off, PAGE, bar);
                    }
                    if (ok2) {
                        const size_t off = static_cast<size_t>(pb2) * block_stride + head_off;
                        bulk_copy_g2s(dst + PAGE, p.kc + off, PAGE, bar);
                        bulk_copy_g2s(dst + 3 * PAGE, p.vc + off, PAGE, bar);
                    }
                } else {
                    mbar_arrive(bar);
                }
                if (!ok || (has2 && !ok2)) atomicOr(p.status, kDevBadBlock);
            }
            const uint32_t bits = (ok ? 1u : 0u) | (ok2 ? 2u : 0u);
            constexpr uint32_t kStageBits = PAIR ? 3u : 1u;
            valid_mask = (valid_mask & ~(kStageBits << (NPG * stage))) | (bits << (NPG * stage));
        };

        const int n_pro = n_my < NS ? n_my : NS;
        for (int i = 0; i < n_pro; ++i) issue(i);

        wa.finish_query(p.scale_log2, k_scale, v_scale);
        wa.reset();

        bool timed_out = false;
        int k = 0;
        for (; k < n_my; ++k) {
            const bool landed = mbar_wait_bounded(bar0 + 8 * stage, phase, p.wait_limit_ns);
            if (!__all_sync(kFull, landed)) {
                timed_out = true;
                break;
            }
            const int jg = j0 + NPG * (warp + W * k);  // the stage's first logical page
            const int valid = ((valid_mask >> (NPG * stage)) & 1u) ? min(B, T - jg * B) : 0;
            const int valid2 =
                (PAIR && ((valid_mask >> (NPG * stage + 1)) & 1u)) ? min(B, T - (jg + 1) * B) : 0;
            const bool full = valid == B && (!PAIR || valid2 == B);
            const uint32_t kbase = wstage0 + static_cast<uint32_t>(stage * STAGE);
            const int pos0 = jg * B - (T - 1);  // ALiBi position of the stage's first slot
            if (!has_alibi) {
                if (full)
                    wa.template page<true, false>(kbase, valid, valid2, pos0);
                else
                    wa.template page<false, false>(kbase, valid, valid2, pos0);
            } else {
                if (full)
                    wa.template page<true, true>(kbase, valid, valid2, pos0);
                else
                    wa.template page<false, true>(kbase, valid, valid2, pos0);
            }
            __syncwarp();
            if (k + NS < n_my) issue(k + NS);
            if (++stage == NS) {
                stage = 0;
                phase ^= 1u;
            }
        }

        if (timed_out) {
            // Let the copies already in flight land (bounded) before the CTA's
            // shared memory can be handed to anyone else, then report.
            const int last = min(n_my, k + NS);
            for (int i = k; i < last; ++i) {
                (void)mbar_wait_bounded(bar0 + 8 * stage, phase, p.wait_limit_ns);
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (lane == 0) atomicOr(p.status, kDevTimeout);
        }

        // ---------------- merge the four warps' partial softmax states
        wa.reduce_l();
        __syncthreads();  // every warp is done with its stages
        float* s_acc = reinterpret_cast<float*>(smem);
        float* s_m = s_acc + W * NH * 8 * RS;
        float* s_l = s_m + W * 16;
        wa.store_merge(s_acc + warp * NH * 8 * RS, RS, s_m + warp * 16, s_l + warp * 16,
                       timed_out);
        __syncthreads();

        const int rows_here = pre ? min(16, rows_total - rg * 16) : p.G;
        const int slot = pre ? part : (cascade ? p.prefix_parts : 0) + part;
        // Balanced: slot 2 c + k of this CTA, G rows (see DecodeParams).
        const long long br_row0 =
            (2LL * blockIdx.x + (bx == bx_first ? 0 : 1)) * static_cast<long long>(p.G);
        for (int idx = threadIdx.x; idx < rows_here * D; idx += (W * 32)) {
            const int h = idx / D;
            const int d = idx - h * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < W; ++w)
                if (s_l[w * 16 + h] > 0.f) M = fmaxf(M, s_m[w * 16 + h]);
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float l = s_l[w * 16 + h];
                if (l > 0.f) {
                    const float wt = exp2f(s_m[w * 16 + h] - M);
                    L += wt * l;
                    O += wt * s_acc[(w * NH * 8 + h) * RS + d];
                }
            }
            const float o = L > 0.f ? (O / L) * wa.out_mul : 0.f;
            const long long row = row_of(h);
            if (direct) {
                p.out[row * D + d] = __float2bfloat16_rn(o);
            } else {
                const long long prow = p.balanced     ? br_row0 + h
                                       : tail_t >= 0 ? (tail_t * p.G + h) * p.tail_P + part
                                                     : row * p.P_total + slot;
                p.ws_o[prow * D + d] = o;
                if (d == 0) {
                    p.ws_m[prow] = M;
                    p.ws_l[prow] = L;
                }
            }
        }
        if (tail_t >= 0) tail_arrive();

        // ---------------- next segment (balanced ranges only)
        if (!p.balanced) break;
        // A barrier every thread reaches: the merge buffer it ends (which overlays
        // the stages) is free again, and a wait that gave up anywhere stops the CTA.
        if (__syncthreads_or(timed_out)) break;
        bx += j1 - j0;
        if (bx >= bx_end) break;
        bj = 0;
        if (++kvh == p.Hk) {
            kvh = 0;
            do {
                ++s;
                bn = pages_of(s);
            } while (bn == 0 && s + 1 < p.S);
        }
    }  // segments
}

struct CombineParams {
    __nv_bfloat16* out;
    const float* ws_o;
    const float* ws_m;
    const float* ws_l;
    const int32_t* seq_lens;
    int S, Hq, P, PP, max_blocks, B;
    int prefix_pages, prefix_parts, P_total;
    int balanced, Hk, G;
    const int* br_scan;  // balanced: per-sequence page prefix [S + 1], pages per CTA
    // Dynamic schedule: every row is merged here from its units' slots --
    // the owners' slots plus one per helper, as the helper counters of the
    // call that just ran (generation hdr[0] - 1) record them.
    int dynamic;
    int dyn_units_pre, dyn_owners, dyn_k_pre, dyn_k_own, dyn_k_total;
    const unsigned int* dyn_hdr;
    const unsigned long long* dyn_uw;
};

// Log-sum-exp merge of the split-KV partials of one (sequence, q head) per
// warp:  M = max_p m_p;  w_p = l_p 2^(m_p - M);  out = sum_p w_p o_p / sum_p w_p.
// Without a shared prefix, rows whose sequence fits in one partition were
// written by the decode kernel and are skipped here.  With one, the slots are
// the prefix partitions followed by the sequence's own partitions.
// Balanced ranges: the unit's pages [off, off + n) were cut over CTAs
// off / per .. (off + n - 1) / per; the first of them holds it in its slot 1
// (its last segment) unless the unit starts its range, every other one in its
// slot 0 (its first segment).  A unit inside one CTA was written by the decode
// kernel; a sequence with no pages gets a zero row here.
// Dynamic schedule: a row's slots are those of its prefix unit (if a prefix
// is declared) followed by those of its (sequence, kv head) unit; every row
// is written here.
// Partitions with an empty sum are skipped.
template <int D>
__global__ void __launch_bounds__(kThreads) pa_combine_kernel(const CombineParams p) {
    grid_dep_wait();  // the decode grid's partials are complete and visible
    grid_dep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto slots_of = [&](int seq, int parts, int pages) {  // non-empty partitions
        const int T = max(0, min(p.seq_lens[seq], p.max_blocks * p.B));
        const int nb = (T + p.B - 1) / p.B;
        return min(parts, (nb + pages - 1) / pages);
    };
    const long long row = (long long)blockIdx.x * kWarps + warp;
    if (row >= (long long)p.S * p.Hq) return;
    const int s = static_cast<int>(row / p.Hq);
    if (!p.dynamic && !p.balanced && p.P_total <= 32) {
        // The row's slots: the prefix partitions, then the sequence's own.
        merge_slots<D>(p.ws_o, p.ws_m, p.ws_l, p.out, row * p.P_total, p.P_total, lane,
                       [&]() -> SlotRow {
            if (p.prefix_pages > 0) {
                const int T = max(0, min(p.seq_lens[s], p.max_blocks * p.B));
                const int nb = (T + p.B - 1) / p.B;
                const int own = nb > p.prefix_pages ? (nb - p.prefix_pages + p.PP - 1) / p.PP : 0;
                return {p.prefix_parts + min(p.P, own), row};
            }
            const int n = slots_of(s, p.P, p.PP);
            return {n <= 1 ? -1 : n, row};  // one partition: the decode kernel wrote the row
        });
        return;
    }
    int nps;
    long long base = row * p.P_total;  // slot i is partial row base + i ...
    long long br_c0 = 0, br_off = 0, br_per = 1;
    int br_g = 0;
    int dyn_n_pre = 0;
    if (p.dynamic) {
        const unsigned int gen = *p.dyn_hdr - 1u;
        const int h = static_cast<int>(row - static_cast<long long>(s) * p.Hq);
        const int kvh = h / p.G;
        auto slots = [&](int u, int k) {
            const unsigned long long w = p.dyn_uw[2 * u + 1];
            const unsigned int helpers =
                static_cast<unsigned int>(w >> 32) == gen ? static_cast<unsigned int>(w) : 0u;
            return p.dyn_owners +
                   static_cast<int>(min(helpers, static_cast<unsigned int>(k - p.dyn_owners)));
        };
        if (p.prefix_pages > 0)
            dyn_n_pre = slots(kvh + p.Hk * ((s * p.G + h % p.G) / 16), p.dyn_k_pre);
        nps = dyn_n_pre + slots(p.dyn_units_pre + s * p.Hk + kvh, p.dyn_k_own);
        base = row * p.dyn_k_total;
    } else if (p.balanced) {
        const int h = static_cast<int>(row - static_cast<long long>(s) * p.Hq);
        const int c_s = __ldg(p.br_scan + s);
        const int n_s = __ldg(p.br_scan + s + 1) - c_s;
        br_per = __ldg(p.br_scan + p.S + 1);
        br_g = h % p.G;
        if (n_s == 0) {
            nps = 0;
        } else {
            br_off = static_cast<long long>(p.Hk) * c_s + static_cast<long long>(h / p.G) * n_s;
            br_c0 = br_off / br_per;
            const long long c1 = (br_off + n_s - 1) / br_per;
            if (c1 == br_c0) return;
            nps = static_cast<int>(c1 - br_c0 + 1);
        }
    } else {
        int T = __ldg(p.seq_lens + s);
        T = max(0, min(T, p.max_blocks * p.B));
        const int nb = (T + p.B - 1) / p.B;
        if (p.prefix_pages > 0) {
            const int own = nb > p.prefix_pages ? (nb - p.prefix_pages + p.PP - 1) / p.PP : 0;
            nps = p.prefix_parts + min(p.P, own);
        } else {
            nps = min(p.P, (nb + p.PP - 1) / p.PP);
            if (nps <= 1) return;
        }
    }
    // ... or, balanced, slot 2 c + k of CTA c = c0 + i, row g of its G rows.
    auto slot_row = [&](int i) -> long long {
        if (p.dynamic) return base + (i < dyn_n_pre ? i : p.dyn_k_pre + (i - dyn_n_pre));
        if (!p.balanced) return base + i;
        const long long c = br_c0 + i;
        const int k = (i == 0 && br_off != br_c0 * br_per) ? 1 : 0;
        return (2 * c + k) * p.G + br_g;
    };
    float M = -INFINITY;
    for (int i = lane; i < nps; i += 32) {
        const long long r = slot_row(i);
        if (p.ws_l[r] > 0.f) M = fmaxf(M, p.ws_m[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    constexpr int PER = D / 32;
    float a[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) a[i] = 0.f;
    float L = 0.f;
    // Slots in groups of 32: each lane loads one slot's (max, sum) and forms
    // its weight, then the group's partial rows are read with the weights
    // broadcast.  Every row is loaded (an empty slot's may hold anything) and
    // an empty slot's contribution is dropped by a select, so the loads of
    // consecutive slots are independent and several are in flight at once.
    for (int i0 = 0; i0 < nps; i0 += 32) {
        const int n = min(32, nps - i0);
        float wt = 0.f;
        long long rl = 0;
        if (lane < n) {
            rl = slot_row(i0 + lane);
            const float l = p.ws_l[rl];
            if (l > 0.f) wt = exp2f(p.ws_m[rl] - M) * l;
        }
        float wsum = wt;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(kFull, wsum, o);
        L += wsum;
#pragma unroll 4
        for (int k = 0; k < n; ++k) {
            const float w = __shfl_sync(kFull, wt, k);
            const long long r = __shfl_sync(kFull, rl, k);
            const float* o = p.ws_o + r * D;
#pragma unroll
            for (int j = 0; j < PER; ++j) {
                const float v = o[lane + 32 * j];
                a[j] += w > 0.f ? w * v : 0.f;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < PER; ++j)
        p.out[row * D + lane + 32 * j] = __float2bfloat16_rn(L > 0.f ? a[j] / L : 0.f);
}

}  // namespace pa
