// Dynamic schedule of the paged decode: persistent CTAs (one wave, every
// resident CTA slot) whose warps keep taking pages of work until none is
// left.
//
// Why: with one CTA per (sequence, kv head, partition) the hardware hands
// units to SMs as they free up, but the last wave runs with part of the GPU
// idle (measured on B200: the whole-GPU rate holds for only 53-92% of a
// call), and equal static shares wait for the slowest SMs (SMs stream pages
// at rates up to ~15% apart).  Here every warp keeps claiming pages while any
// are left, in claims that shrink as a unit runs out, so the GPU stays busy
// to the end.  This is the persistent, resident-CTA way of running the
// decode that "Why PagedAttention was retired", section 5, lists among the
// capabilities the legacy kernel gave up.
//
// Units are (sequence, kv head) pairs, after the shared-prefix units (kv
// head, group of 16 query rows) when a prefix is declared.  Each unit has a
// page counter in the workspace.  A cursor hands every unit to `owners`
// warps (partial slots 0 .. owners - 1): four for a batch with at least
// half as many units as warps, as the four warps of a CTA share a unit in
// pa_decode_kernel, else one.  A warp claims ranges of its unit's pages from
// the unit's counter -- each range a quarter of the pages left, 4 to 32
// ring stages -- and accumulates every page it reads in registers.  When its unit is exhausted it takes the next cursor entry; once
// the cursor is spent, it joins as a helper (the next slots; at most K slots
// per unit) the unit with the most pages left per warp on it, until no unit
// has pages worth joining for.  Each (warp, unit) pair writes one fp32
// partial (o = acc / l, max, sum) and pa_combine_kernel merges a row's
// slots.  So a row has as many partials as warps read its unit: one for most
// units of a large batch, about total warps / units for a few long ones.
//
// Each warp is an independent producer/consumer pipeline: lane 0 copies
// whole K and V pages into the warp's ring of shared-memory stages (1-D bulk
// async copies completing on the stage's mbarrier), and the next range's
// claim is made while the current one is issued, so the ring keeps flowing
// across range and unit ends.  Each stage records the unit, slot and page
// it holds; the consumer finishes a unit when the next stage belongs to
// another.  Warps share no shared memory, take no block barrier and never
// wait for one another.
//
// Counters: a generation number, the unit cursor and a count of finished
// warps sit in the workspace header (bytes 64..75); each unit's page and
// helper counters are 64-bit words (generation << 32 | count), so a word
// left by an earlier call reads as zero and nothing needs clearing between
// calls.  The last warp to finish moves the generation on and puts the
// cursor and the count back to zero.  Every wait is bounded as in
// pa_decode_kernel; a warp whose wait gives up drains its copies, writes
// empty partials for the units it holds, sets PA_DEV_WAIT_TIMEOUT and stops.
#pragma once

#include "pa_decode_kernels.cuh"

namespace pa {

constexpr int kDynHeaderWord = 16;  // first of the dynamic schedule's header words (byte 64)

struct DynParams {
    int units_pre;    // shared-prefix units (0 without a prefix), numbered first
    int units;        // units_pre + num_seqs * num_kv_heads
    int owners;       // warps the cursor hands each unit to (slots 0 .. owners - 1)
    int k_pre, k_own;  // partial slots per row of a prefix / per-sequence unit
    int k_total;       // k_pre + k_own: slots per query row (prefix slots first)
    int total_warps;   // warps of the grid
    int step_min, step_max;  // pages per claim
    int probe_rounds;        // 32-unit rounds a warp probes when looking for a unit to help
    unsigned int* hdr;       // [0] generation, [1] unit cursor, [2] warps finished
    unsigned long long* uw;  // [units][2]: page counter, helper counter
};

// A unit's place in the batch: prefix unit (kv head, row group) or
// (sequence, kv head); its pages in the block-table row; its tokens (clamped
// as pa_decode_kernel clamps them) and the range-check bits found.
struct UnitRef {
    int u;
    bool pre;
    int kvh, s, rg;
    int j_base, n;  // pages j_base .. j_base + n - 1 of the row
    int T;
    uint32_t bad;
};

template <int B>
__device__ __forceinline__ UnitRef unit_ref(const DecodeParams& p, const DynParams& t, int u) {
    UnitRef r;
    r.u = u;
    r.bad = 0;
    if (u < t.units_pre) {
        r.pre = true;
        r.kvh = u % p.Hk;
        r.rg = u / p.Hk;
        r.s = 0;
        r.j_base = 0;
        r.n = p.prefix_pages;
        r.T = p.prefix_pages * B;
    } else {
        const int v = u - t.units_pre;
        r.pre = false;
        r.kvh = v % p.Hk;
        r.s = v / p.Hk;
        r.rg = 0;
        const int t_cap = p.max_blocks * B;
        int T = __ldg(p.seq_lens + r.s);
        if (T < 0) { T = 0; r.bad = kDevSeqLen; }
        if (T > t_cap) { T = t_cap; r.bad = kDevSeqLen; }
        if (p.prefix_pages > 0 && T < p.prefix_pages * B) r.bad |= kDevPrefix;
        r.T = T;
        r.j_base = p.prefix_pages;
        r.n = max(0, (T + B - 1) / B - p.prefix_pages);
    }
    return r;
}

// Count of a generation-tagged counter word (0 when the word is from
// another generation).
__device__ __forceinline__ uint32_t tagged_count(unsigned long long w, uint32_t gen) {
    return static_cast<uint32_t>(w >> 32) == gen ? static_cast<uint32_t>(w) : 0u;
}

// Add `step` to a generation-tagged counter, bringing a word left by an
// earlier call to this generation first; returns the count before the add,
// or 0xffffffff if the compare-and-swap never succeeded (bounded).
__device__ __forceinline__ uint32_t tagged_add(unsigned long long* w, uint32_t gen, uint32_t step) {
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(w);
    for (int it = 0; it < (1 << 20); ++it) {
        const uint32_t v = tagged_count(cur, gen);
        const unsigned long long nw = (static_cast<unsigned long long>(gen) << 32) | (v + step);
        const unsigned long long prev = atomicCAS(w, cur, nw);
        if (prev == cur) return v;
        cur = prev;
    }
    return 0xffffffffu;
}

// SC: one query head per kv head on the CUDA cores (WarpAttnScalar).
template <int D, int B, bool FP8, int NH, int W, bool F8MMA, bool SC = false>
__global__ void __launch_bounds__(W * 32,
                                  ((pair_pages<D, B, FP8, F8MMA>() && !F8MMA && NH == 1) || SC) ? 3
                                                                                                : 1)
    pa_decode_dyn_kernel(const DecodeParams p, const __grid_constant__ DynParams t) {
    static_assert(!F8MMA || FP8, "e4m3 MMAs need e4m3 pages");
    static_assert(!SC || (!FP8 && NH == 1), "the CUDA-core form takes bf16 pages and one head");
    using WA = std::conditional_t<SC, WarpAttnScalar<D, B>, WarpAttn<D, B, FP8, NH, F8MMA>>;
    constexpr int PAGE = WA::PAGE;
    constexpr int NPG = WA::NPG;
    constexpr bool PAIR = WA::PAIR;
    constexpr int STAGE = 2 * PAGE * NPG;

    extern __shared__ __align__(128) uint8_t smem[];

    // Programmatic dependent launch: nothing is touched before the grid ahead
    // in the stream (the previous call, or whatever wrote the inputs) is done.
    grid_dep_wait();
    grid_dep_launch_dependents();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * W + warp;  // this warp's number in the grid

    // Shared memory: per-warp page stages, then the mbarriers, then each
    // stage's record (unit, slot, first page).
    const int NS = p.stages;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t wstage0 = sbase + static_cast<uint32_t>(warp * NS * STAGE);
    const uint32_t bar0 = sbase + static_cast<uint32_t>(W * NS * STAGE + warp * NS * 8);
    int* meta = reinterpret_cast<int*>(smem + W * NS * STAGE + W * NS * 8) + warp * NS * 4;
    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint32_t gen = *reinterpret_cast<volatile unsigned int*>(t.hdr);
    const bool cascade = p.prefix_pages > 0;
    const int rows_total = p.S * p.G;
    const size_t block_stride = static_cast<size_t>(p.Hk) * PAGE;
    float k_scale = 1.f, v_scale = 1.f;
    if constexpr (FP8) {
        k_scale = __ldg(p.k_scale);
        v_scale = __ldg(p.v_scale);
    }
    const bool has_alibi = p.alibi != nullptr;

    // Query row (s * Hq + head) of local row lr of a unit, or -1.
    auto row_of = [&](const UnitRef& r, int lr) -> long long {
        if (r.pre) {
            const int gi = r.rg * 16 + lr;
            if (gi >= rows_total) return -1;
            return (long long)(gi / p.G) * p.Hq + (long long)r.kvh * p.G + gi % p.G;
        }
        return lr < p.G ? (long long)r.s * p.Hq + (long long)r.kvh * p.G + lr : -1;
    };
    auto rows_of = [&](const UnitRef& r) { return r.pre ? min(16, rows_total - r.rg * 16) : p.G; };
    // Partial row of (query row, unit kind, slot): the prefix's slots first.
    auto prow_of = [&](long long row, bool pre, int slot) -> long long {
        return row * t.k_total + (pre ? slot : t.k_pre + slot);
    };
    // An empty partial (sum 0) for every row of (unit, slot): the combine
    // skips it.
    auto empty_partial = [&](const UnitRef& r, int slot) {
        const int n = rows_of(r);
        for (int h = lane; h < n; h += 32) {
            const long long prow = prow_of(row_of(r, h), r.pre, slot);
            p.ws_m[prow] = -INFINITY;
            p.ws_l[prow] = 0.f;
        }
    };

    // ------------------------------------------------------------ producer
    UnitRef iu;            // unit being issued
    iu.u = -1;
    int islot = 0;         // this warp's slot in it
    const int32_t* ibt = p.bt;
    size_t ihead = 0;
    int ra = 0, rn = 0, ri = 0;  // current range: pages ra .. ra + NPG * rn of the unit, next stage ri
    int win_a = -1, win_a2 = -1;  // block ids of the current range: lane l <-> stage l
    int win_n = -1, win_n2 = -1;  // ... and of the next range, once loaded
    int nv = 0, nstep = 0;         // the next range's claim (count before it, pages)
    int nv_b = 0;                  // its count, once read
    bool n_claimed = false;        // a next-range claim is in flight
    bool n_loaded = false;         // the next range's block ids are in win_n
    bool cursor_done = false, exhausted = false;
    uint32_t valid_mask = 0;  // bit NPG * stage (+ 1): that page had a legal block id

    auto claim_step = [&](int left) {
        int st = left / 4;
        st = max(t.step_min, min(t.step_max, st));
        return (st + NPG - 1) / NPG * NPG;
    };
    // Block ids of range [v, v + step) of the current unit: lane l <-> stage l.
    auto load_window = [&](int v, int step, int& w1, int& w2) {
        const int n_stages = (min(v + step, iu.n) - v + NPG - 1) / NPG;
        const int j = iu.j_base + v + NPG * lane;
        const int jend = iu.j_base + iu.n;
        w1 = (lane < n_stages && j < jend) ? __ldg(ibt + j) : -1;
        if constexpr (PAIR) w2 = (lane < n_stages && j + 1 < jend) ? __ldg(ibt + j + 1) : -1;
    };
    // Start issuing range [v, v + step) of the current unit (clipped to it);
    // false when the unit has no pages there.  `preloaded`: its block ids are
    // in win_n already.
    auto start_range = [&](int v, int step, bool preloaded) -> bool {
        if (v >= iu.n) return false;
        ra = v;
        rn = (min(v + step, iu.n) - v + NPG - 1) / NPG;
        ri = 0;
        if (preloaded) {
            win_a = win_n;
            win_a2 = win_n2;
        } else {
            load_window(ra, step, win_a, win_a2);
        }
        // Claim the range after this one now; its count is read when this
        // range runs out, so the atomic's latency is hidden.
        nstep = claim_step(iu.n - (v + step));
        if (lane == 0) {
            const unsigned long long w = atomicAdd(t.uw + 2 * iu.u, static_cast<unsigned long long>(nstep));
            nv = static_cast<int>(static_cast<uint32_t>(w));
        }
        n_claimed = true;
        n_loaded = false;
        return true;
    };
    // Join unit u with slot `slot`: claim its first range.  A unit with no
    // pages left gets an empty partial for the slot.
    auto join = [&](int u, int slot) -> bool {
        iu = unit_ref<B>(p, t, u);
        islot = slot;
        ibt = p.bt + (iu.pre ? 0 : (long long)iu.s * p.max_blocks);
        ihead = static_cast<size_t>(iu.kvh) * PAGE;
        if (slot == 0 && !iu.pre && iu.kvh == 0) {  // the first owner checks the sequence once
            if (iu.bad && lane == 0) atomicOr(p.status, iu.bad);
            if (cascade && iu.s > 0) {
                // The declared prefix must be the same physical blocks as row 0's.
                bool same = true;
                for (int j = lane; j < p.prefix_pages; j += 32)
                    same &= __ldg(ibt + j) == __ldg(p.bt + j);
                if (!__all_sync(kFull, same) && lane == 0) atomicOr(p.status, kDevPrefix);
            }
        }
        const int step = claim_step(iu.n);
        uint32_t v = 0;
        if (lane == 0) v = tagged_add(t.uw + 2 * u, gen, static_cast<uint32_t>(step));
        v = __shfl_sync(kFull, v, 0);
        if (v == 0xffffffffu) {  // the counter could not be updated: give the unit up
            if (lane == 0) atomicOr(p.status, kDevTimeout);
            v = static_cast<uint32_t>(iu.n);
        }
        if (!start_range(static_cast<int>(v), step, false)) {
            empty_partial(iu, slot);
            iu.u = -1;
            return false;
        }
        // Warm L2 with the unit's query rows for the consumer.
        const long long qr = row_of(iu, lane >> 1);
        if ((lane >> 1) < rows_of(iu) && qr >= 0) prefetch_l2(p.q + qr * D + (lane & 1) * (D / 2));
        return true;
    };
    // The unit to help: among the units probed with at least two minimum
    // claims of pages left, the one with the most pages left per warp already
    // on it (owner plus helpers), so that warps looking at the same time
    // spread over the units instead of piling onto one; it must have a free
    // helper slot.  Gives up after four probes that find nothing worth
    // joining, or 16 tries in all.
    auto help = [&]() -> bool {
        int empty = 0;
        for (int attempt = 0; attempt < 16; ++attempt) {
            const unsigned int h = (static_cast<unsigned int>(gw) * 2654435761u) ^ (attempt * 40503u);
            int best_u = -1;
            float best_score = 0.f;
            for (int k = 0; k < t.probe_rounds; ++k) {
                const int u = static_cast<int>((h + static_cast<unsigned int>(lane + 32 * k)) %
                                               static_cast<unsigned int>(t.units));
                const UnitRef r = unit_ref<B>(p, t, u);
                const volatile unsigned long long* w =
                    reinterpret_cast<volatile unsigned long long*>(t.uw + 2 * u);
                const int used = static_cast<int>(tagged_count(w[0], gen));
                const int helpers = static_cast<int>(tagged_count(w[1], gen));
                const int left = r.n - used;
                const int k_max = u < t.units_pre ? t.k_pre : t.k_own;
                if (left >= 2 * t.step_min && t.owners + helpers < k_max) {
                    const float score = static_cast<float>(left) / static_cast<float>(2 + helpers);
                    if (score > best_score) {
                        best_score = score;
                        best_u = u;
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float os = __shfl_xor_sync(kFull, best_score, o);
                const int ou = __shfl_xor_sync(kFull, best_u, o);
                if (os > best_score || (os == best_score && ou > best_u)) {
                    best_score = os;
                    best_u = ou;
                }
            }
            if (best_u < 0) {  // nothing worth joining among these units
                if (++empty == 4) return false;
                continue;
            }
            const int k_max = best_u < t.units_pre ? t.k_pre : t.k_own;
            uint32_t hs = 0;
            if (lane == 0) hs = tagged_add(t.uw + 2 * best_u + 1, gen, 1u);
            hs = __shfl_sync(kFull, hs, 0);
            if (hs == 0xffffffffu || t.owners + static_cast<int>(hs) >= k_max) continue;  // no slot
            if (join(best_u, t.owners + static_cast<int>(hs))) return true;
        }
        return false;
    };
    // The next unit: from the cursor while it lasts (entry e is owner slot
    // e % owners of unit e / owners), then one to help.
    auto next_unit = [&]() -> bool {
        while (!cursor_done) {
            unsigned int e = 0;
            if (lane == 0) e = atomicAdd(t.hdr + 1, 1u);
            e = __shfl_sync(kFull, e, 0);
            if (e >= static_cast<unsigned int>(t.units) * static_cast<unsigned int>(t.owners)) {
                cursor_done = true;
                break;
            }
            if (join(static_cast<int>(e / t.owners), static_cast<int>(e % t.owners))) return true;
        }
        return help();
    };

    // Issue the next stage of work into ring stage `st`; false when no work
    // is left for this warp.
    auto issue_next = [&](int st) -> bool {
        if (exhausted) return false;
        while (iu.u < 0 || ri >= rn) {
            bool ok = false;
            if (iu.u >= 0 && n_claimed) {  // the current unit's next range
                n_claimed = false;
                const int v = n_loaded ? nv_b : __shfl_sync(kFull, nv, 0);
                ok = start_range(v, nstep, n_loaded);
            }
            if (!ok) {
                iu.u = -1;
                if (!next_unit()) {
                    exhausted = true;
                    return false;
                }
            }
        }
        const int i = ri++;
        // Halfway through a range the next range's claim (an atomic issued
        // when this range started) has long returned: read it and load its
        // block ids now, so they are in registers when this range runs out.
        // (Reading it sooner would stall the warp on the atomic's latency.)
        if (n_claimed && !n_loaded && i == rn / 2) {
            nv_b = __shfl_sync(kFull, nv, 0);
            if (nv_b < iu.n) load_window(nv_b, nstep, win_n, win_n2);
            n_loaded = true;
        }
        const int jg = iu.j_base + ra + NPG * i;  // the stage's first page in the row
        const int pb = __shfl_sync(kFull, win_a, i);
        const int pb2 = PAIR ? __shfl_sync(kFull, win_a2, i) : -1;
        const uint32_t bar = bar0 + 8 * st;
        const bool ok = pb >= 0 && static_cast<long long>(pb) < p.num_blocks;
        const bool has2 = PAIR && jg + 1 < iu.j_base + iu.n;
        const bool ok2 = has2 && pb2 >= 0 && static_cast<long long>(pb2) < p.num_blocks;
        if (lane == 0) {
            meta[4 * st] = iu.u;
            meta[4 * st + 1] = islot;
            meta[4 * st + 2] = jg;
            const uint32_t bytes = (ok ? 2 * PAGE : 0) + (ok2 ? 2 * PAGE : 0);
            const uint32_t dst = wstage0 + static_cast<uint32_t>(st * STAGE);
            if (bytes) {
                mbar_arrive_expect_tx(bar, bytes + p.stall_tx_bytes);
                if (ok) {
                    const size_t off = static_cast<size_t>(pb) * block_stride + ihead;
                    bulk_copy_g2s(dst, p.kc + off, PAGE, bar);
                    bulk_copy_g2s(dst + NPG * PAGE, p.vc + off, PAGE, bar);
                }
                if (ok2) {
                    const size_t off = static_cast<size_t>(pb2) * block_stride + ihead;
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
        valid_mask = (valid_mask & ~(kStageBits << (NPG * st))) | (bits << (NPG * st));
        return true;
    };

    // ------------------------------------------------------------ consumer
    WA wa(lane);
    UnitRef cu;  // unit being consumed
    cu.u = -1;
    int cslot = 0;

    auto begin_unit = [&](int u, int slot) {
        cu = unit_ref<B>(p, t, u);
        cslot = slot;
        auto rows = [&](int lr) { return row_of(cu, lr); };
        wa.fetch_query(p.q, rows);
        wa.set_alibi(p.alibi, p.Hq, rows);
        wa.finish_query(p.scale_log2, k_scale, v_scale);
        wa.reset();
    };

    // The unit's partial for this warp's slot: o = acc / l (times the output
    // multiplier) and (max, sum); `dead` leaves an empty partial instead.
    auto finish_unit = [&](bool dead) {
        wa.write_partial(p.ws_o, p.ws_m, p.ws_l, rows_of(cu),
                         [&](int h) { return prow_of(row_of(cu, h), cu.pre, cslot); }, dead);
    };

    // ------------------------------------------------------------ the ring
    int stage = 0, issue_stage = 0, pending = 0;
    uint32_t phase = 0;
    for (int i = 0; i < NS; ++i) {
        if (!issue_next(issue_stage)) break;
        issue_stage = (issue_stage + 1 == NS) ? 0 : issue_stage + 1;
        ++pending;
    }
    __syncwarp();

    bool timed_out = false;
    while (pending > 0) {
        const bool landed = mbar_wait_bounded(bar0 + 8 * stage, phase, p.wait_limit_ns);
        if (!__all_sync(kFull, landed)) {
            timed_out = true;
            break;
        }
        const int u = meta[4 * stage];
        const int slot = meta[4 * stage + 1];
        const int jg = meta[4 * stage + 2];
        if (u != cu.u || slot != cslot) {
            if (cu.u >= 0) finish_unit(false);
            begin_unit(u, slot);
        }
        const int T = cu.T;
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
        __syncwarp();  // every lane is done with the stage before it is refilled
        --pending;
        if (issue_next(issue_stage)) {
            issue_stage = (issue_stage + 1 == NS) ? 0 : issue_stage + 1;
            ++pending;
        }
        __syncwarp();
        if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
        }
    }

    if (!timed_out) {
        if (cu.u >= 0) finish_unit(false);
    } else {
        // Let the copies in flight land (bounded), then leave empty partials
        // for every (unit, slot) this warp holds: the one being consumed,
        // those waiting in the ring, and the one being issued.
        int last_u = cu.u, last_slot = cslot;
        if (cu.u >= 0) finish_unit(true);
        for (int k = 0; k < pending; ++k) {
            (void)mbar_wait_bounded(bar0 + 8 * stage, phase, p.wait_limit_ns);
            const int u = meta[4 * stage];
            const int slot = meta[4 * stage + 1];
            if (u != last_u || slot != last_slot) {
                empty_partial(unit_ref<B>(p, t, u), slot);
                last_u = u;
                last_slot = slot;
            }
            if (++stage == NS) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (iu.u >= 0 && (iu.u != last_u || islot != last_slot)) empty_partial(iu, islot);
        if (lane == 0) atomicOr(p.status, kDevTimeout);
    }

    // The last warp to finish moves the generation on and puts the cursor
    // and the count of finished warps back to zero for the next call (every
    // counter of this call has been used by then).
    if (lane == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(t.hdr + 2, 1u);
        if (prev == static_cast<unsigned int>(t.total_warps) - 1u) {
            atomicExch(t.hdr + 1, 0u);
            atomicExch(t.hdr + 2, 0u);
            atomicAdd(t.hdr, 1u);
        }
    }
}

}  // namespace pa
