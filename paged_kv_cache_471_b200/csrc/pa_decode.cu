// C ABI of libpagedattn: argument checks, the split-KV planner, and the
// launches of pa_decode_kernel / pa_combine_kernel.  See include/pagedattn.h
// for the contract of each entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "pa_decode_dynamic.cuh"
#include "pa_decode_kernels.cuh"
#include "pagedattn.h"

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr size_t kSmemPerSm = 228 * 1024;
constexpr size_t kSmemReservedPerCta = 1024;
constexpr size_t kMaxSmemPerCta = 227 * 1024;  // opt-in limit of sm_100
constexpr size_t kStaticSmemReserve = 256;      // the kernel's own __shared__ variables
constexpr int kMinPartitionPages = 16;
constexpr int kMaxRankedSeqs = 256;  // batches ranked by length on the device
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // a page copy's wait bound
constexpr unsigned long long kTestWaitLimitNs = 20000000ull;  // with test_stall_copies
constexpr long long kLongPartitionPages = 256;
// Partials per query row that the combine kernel merges with one batch of
// loads (a slot per lane); split plans keep to it where they can.
constexpr long long kOneBatchSlots = 32;
// CTAs of a split plan for a batch of only a handful of (sequence, kv head)
// units, where one partial wave within kOneBatchSlots would stay small:
// kFewUnitCtas per kFewUnitSms SMs (128 on a 148-SM B200), scaled to the SMs
// the plan is made for.
constexpr long long kFewUnitCtas = 128;
constexpr long long kFewUnitSms = 148;
// Split tail: partitions per unit of the last, partial wave of whole units
// (at least; more when that wave has few units, up to kMaxTailParts).
constexpr int kTailParts = 4;
constexpr int kMaxTailParts = 16;
// Workspace layout: the header (status word, dynamic-schedule words), then
// the split tail's per-unit merge counts, which nothing else touches (they
// are 0 between calls), then the plan's partials (or page scan, or unit
// counters).
constexpr long long kMergeCounts = PA_WORKSPACE_MERGE_COUNT_BYTES / sizeof(unsigned int);
constexpr size_t kBodyOffset = PA_WORKSPACE_HEADER_BYTES + PA_WORKSPACE_MERGE_COUNT_BYTES;
constexpr int kDefaultStages = 2;
constexpr int kMaxShortStages = 4;
constexpr size_t kShortStagesSmem = 96 * 1024;  // keep >= 2 CTAs per SM
constexpr long long kMaxCtasPerSm = 3;
constexpr int kMaxForcedStages = 16;
constexpr int kMaxDevices = 64;
constexpr long long kMaxDynSlots = 64;  // partial slots per row and unit kind (dynamic schedule)

thread_local char g_detail[256] = "";

pa_status fail(pa_status st, const char* fmt, const char* what) {
    std::snprintf(g_detail, sizeof g_detail, fmt, what);
    return st;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

int elem_bytes(pa_kv_dtype t) { return t == PA_KV_FP8_E4M3 ? 1 : 2; }

pa_status check_sizes(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                      int block_size, int max_seq_len, pa_kv_dtype kv_dtype) {
    if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "%s", "num_seqs < 0");
    if (num_heads <= 0 || num_kv_heads <= 0)
        return fail(PA_ERR_INVALID_ARG, "%s", "num_heads and num_kv_heads must be > 0");
    if (num_heads % num_kv_heads)
        return fail(PA_ERR_INVALID_ARG, "%s", "num_heads must be a multiple of num_kv_heads");
    if (num_heads / num_kv_heads > 16)
        return fail(PA_ERR_UNSUPPORTED, "%s", "num_heads / num_kv_heads > 16");
    if (head_size != 64 && head_size != 128)
        return fail(PA_ERR_UNSUPPORTED, "%s", "head_size must be 64 or 128");
    if (block_size != 16 && block_size != 32)
        return fail(PA_ERR_UNSUPPORTED, "%s", "block_size must be 16 or 32");
    if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3)
        return fail(PA_ERR_UNSUPPORTED, "%s", "kv_dtype");
    if (max_seq_len < 0) return fail(PA_ERR_INVALID_ARG, "%s", "max_seq_len < 0");
    return PA_OK;
}

int device_sms(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    static std::atomic<int> cache[kMaxDevices];
    if (dev >= 0 && dev < kMaxDevices) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) {
            *out = v;
            return 0;
        }
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return -1;
    if (dev >= 0 && dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    *out = n;
    return 0;
}

size_t merge_bytes(int head_size, int group, int warps) {
    const int nh = group > 8 ? 2 : 1;
    return static_cast<size_t>(warps * nh * 8 * (head_size + 4) + 2 * warps * 16) * 4;
}

pa_status plan(pa_plan* pl, int num_seqs, int num_heads, int num_kv_heads, int head_size,
               int block_size, int max_seq_len, pa_kv_dtype kv_dtype, const pa_options* opts) {
    pa_status st = check_sizes(num_seqs, num_heads, num_kv_heads, head_size, block_size,
                               max_seq_len, kv_dtype);
    if (st != PA_OK) return st;
    int sms = opts ? opts->num_sms : 0;
    if (sms < 0) return fail(PA_ERR_INVALID_ARG, "%s", "opts->num_sms < 0");
    if (opts && opts->partition_pages < 0)
        return fail(PA_ERR_INVALID_ARG, "%s", "opts->partition_pages < 0");
    if (sms == 0 && device_sms(&sms) != 0)
        return fail(PA_ERR_CUDA, "%s", "cannot query the SM count of the current device");

    if (opts && (opts->stages < 0 || opts->stages == 1 || opts->stages > kMaxForcedStages))
        return fail(PA_ERR_INVALID_ARG, "%s", "opts->stages must be 0 or 2..16");
    // Two page buffers per warp: measured on B200, more resident CTAs beat
    // deeper per-warp rings for the same bytes in flight.
    const int prefix = opts ? opts->shared_prefix_blocks : 0;
    if (prefix < 0 || static_cast<long long>(prefix) * block_size > max_seq_len)
        return fail(PA_ERR_INVALID_ARG, "%s",
                    "opts->shared_prefix_blocks must be in [0, max_seq_len / block_size]");
    const bool cascade = prefix > 0 && num_seqs > 0;
    if (cascade && opts->alibi_slopes)
        return fail(PA_ERR_UNSUPPORTED, "%s", "ALiBi slopes with a shared prefix");
    const int schedule = opts ? opts->schedule : PA_SCHEDULE_AUTO;
    if (schedule != PA_SCHEDULE_AUTO && schedule != PA_SCHEDULE_BALANCED &&
        schedule != PA_SCHEDULE_PARTITIONED && schedule != PA_SCHEDULE_DYNAMIC)
        return fail(PA_ERR_INVALID_ARG, "%s", "opts->schedule");
    const bool f8mma = opts && opts->fp8_compute && kv_dtype == PA_KV_FP8_E4M3;
    // A stage holds a K and a V page; small pages (16-token e4m3 pages, and
    // 16-token bf16 pages of head size 64) go in pairs (pa_decode_kernels.cuh,
    // pair_pages).
    const bool pair = block_size == 16 && (kv_dtype == PA_KV_FP8_E4M3 || head_size == 64);
    const size_t stage = 2ull * head_size * block_size * elem_bytes(kv_dtype) * (pair ? 2 : 1);
    const int W = pa::decode_warps(static_cast<long long>(stage));
    int ns = kDefaultStages;
    if (opts && opts->stages > 0) ns = opts->stages;
    size_t stage_area = static_cast<size_t>(W) * ns * stage;
    const size_t mb = merge_bytes(head_size, cascade ? 16 : num_heads / num_kv_heads, W);
    if (stage_area < mb) stage_area = mb;
    // After the stages: a page mbarrier per buffer; with a shared prefix also
    // the prefix units' shared ring's "empty" mbarriers and page flags.
    const size_t bar_bytes_per_buffer = cascade ? 24 : 8;
    size_t smem = stage_area + static_cast<size_t>(W) * ns * bar_bytes_per_buffer;
    if (smem > kMaxSmemPerCta - kStaticSmemReserve)
        return fail(PA_ERR_INVALID_ARG, "%s", "too many stages for shared memory");
    long long per_sm = static_cast<long long>(kSmemPerSm / (smem + kSmemReservedPerCta));
    if (per_sm < 1) per_sm = 1;
    if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;  // register limit
    if (f8mma && per_sm > 2) per_sm = 2;                // e4m3-MMA forms: ~200+ registers
    const long long slots = static_cast<long long>(sms) * per_sm;

    const long long pages_max = (static_cast<long long>(max_seq_len) + block_size - 1) / block_size;
    const long long units = static_cast<long long>(num_seqs) * num_kv_heads;

    // Balanced ranges (on request): one wave of CTAs, each an equal share of
    // all pages (pa_decode_kernels.cuh).  Not the default: measured on B200,
    // SMs stream bf16 pages at rates ~7% apart (std), so equal static shares
    // wait for the slowest SMs, while one CTA per unit lets the hardware hand
    // more units to faster SMs.  e4m3 pages stream at even rates across SMs,
    // and there the balanced ranges gained ~1% (256 x 16384 tokens).  Needs no
    // shared prefix, no forced partitions, the per-sequence page scan in the
    // stage area, and page counts in int.
    const bool forced_pp = opts && opts->partition_pages > 0;
    pl->dynamic = 0;
    pl->tail_units = 0;
    pl->tail_partitions = 0;
    pl->tail_partition_pages = 0;
    pl->combine = 0;
    pl->longest_first = 0;
    if (schedule == PA_SCHEDULE_DYNAMIC) {
        // Persistent warps claiming pages (pa_decode_dynamic.cuh): one wave of
        // CTAs; per query row, a slot per warp that read its unit (at most
        // kslots), for the prefix unit and the row's own unit.
        if (forced_pp)
            return fail(PA_ERR_UNSUPPORTED, "%s", "the dynamic schedule takes no forced partitions");
        const long long groups =
            cascade ? (static_cast<long long>(num_seqs) * (num_heads / num_kv_heads) + 15) / 16 : 0;
        const long long units_pre = static_cast<long long>(num_kv_heads) * groups;
        const long long n_units = units_pre + units;
        if (n_units >= (1ll << 30) || static_cast<long long>(num_seqs) * num_heads >= (1ll << 31))
            return fail(PA_ERR_INVALID_ARG, "%s", "batch too large for the dynamic schedule");
        // Owners per unit: four when the batch has at least half as many units
        // as warps (the four warps of a CTA per unit of the partitioned
        // schedule), else one.  Slots per unit: the owners', and enough
        // helpers that the last units can take every warp (twice the warps
        // per unit, plus 8).
        const long long warps = slots * W;
        const long long owners = 2 * n_units >= warps ? 4 : 1;
        long long kslots = n_units > 0 ? owners + (2 * warps + n_units - 1) / n_units + 8 : 2;
        if (kslots > kMaxDynSlots) kslots = kMaxDynSlots;
        const long long k_total = (cascade ? 2 : 1) * kslots;
        const size_t dsmem = static_cast<size_t>(W) * ns * (stage + 8 + 16);
        if (dsmem > kMaxSmemPerCta - kStaticSmemReserve)
            return fail(PA_ERR_INVALID_ARG, "%s", "too many stages for shared memory");
        size_t ws = kBodyOffset;
        ws += (static_cast<size_t>(n_units) * 16 + 255) & ~static_cast<size_t>(255);
        ws += static_cast<size_t>(num_seqs) * num_heads * k_total *
              (static_cast<size_t>(head_size) + 2) * sizeof(float);
        ws = (ws + 255) & ~static_cast<size_t>(255);
        pl->num_partitions = static_cast<int>(kslots);
        pl->partition_pages = 0;
        pl->stages = ns;
        pl->warps_per_cta = W;
        pl->grid_ctas = slots;
        pl->smem_bytes = dsmem;
        pl->workspace_bytes = ws;
        pl->prefix_partitions = cascade ? static_cast<int>(kslots) : 0;
        pl->prefix_groups = static_cast<int>(groups);
        pl->balanced = 0;
        pl->dynamic = static_cast<int>(owners);
        pl->combine = 1;
        return PA_OK;
    }
    const bool br_fits = !cascade && !forced_pp && num_seqs > 0 &&
                         (static_cast<size_t>(num_seqs) + 1 + 32 * W) * 4 <= stage_area &&
                         units * (pages_max + 1) < (1ll << 31);
    if (schedule == PA_SCHEDULE_BALANCED && !br_fits)
        return fail(PA_ERR_UNSUPPORTED, "%s",
                    "balanced ranges need no shared prefix, no forced partitions and a batch "
                    "whose lengths fit the stage memory");
    const bool balanced = br_fits && schedule == PA_SCHEDULE_BALANCED;
    if (balanced) {
        const long long rows = 2 * slots * (num_heads / num_kv_heads);
        size_t ws = kBodyOffset;
        ws += ((static_cast<size_t>(num_seqs) + 2) * sizeof(int) + 255) & ~static_cast<size_t>(255);
        ws += static_cast<size_t>(rows) * (static_cast<size_t>(head_size) + 2) * sizeof(float);
        ws = (ws + 255) & ~static_cast<size_t>(255);
        pl->num_partitions = 0;
        pl->partition_pages = 0;
        pl->stages = ns;
        pl->warps_per_cta = W;
        pl->grid_ctas = slots;
        pl->smem_bytes = smem;
        pl->workspace_bytes = ws;
        pl->prefix_partitions = 0;
        pl->prefix_groups = 0;
        pl->balanced = 1;
        pl->combine = 1;
        return PA_OK;
    }
    long long pp;
    bool whole_units = false;  // at least two waves of units, none split
    if (opts && opts->partition_pages > 0) {
        pp = opts->partition_pages;
    } else if (pages_max == 0 || units == 0) {
        pp = 1;
    } else if (units >= 2 * slots && num_seqs <= kMaxRankedSeqs) {
        // At least two waves of (sequence, kv head) units: no split.  CTAs
        // take sequences longest first (ranked on the device), which keeps
        // the last wave short for mixed lengths.  Between one and two waves,
        // equal lengths would leave a last wave of a few full-length units
        // running alone, so those batches are split (measured on B200: 64
        // sequences x 8 kv heads x 16384 tokens ran 12% slower unsplit).
        pp = pages_max;
        whole_units = true;
    } else {
        // Split count:
        //  * enough partitions to balance uneven lengths: about four partitions
        //    of work per CTA slot if every sequence were max_seq_len long, each
        //    at least kMinPartitionPages;
        //  * but no partition shorter than kLongPartitionPages unless that is
        //    needed to give every CTA slot a partition (long partitions
        //    amortise each CTA's start-up and merge; measured on B200).
        const long long per_slot = (units * pages_max + slots - 1) / slots;
        long long target = (per_slot + 3) / 4;
        if (target < kMinPartitionPages) target = kMinPartitionPages;
        const long long p_bal = (pages_max + target - 1) / target;
        const long long p_fill = (slots + units - 1) / units;
        const long long p_long = pages_max / kLongPartitionPages > 1 ? pages_max / kLongPartitionPages : 1;
        long long np = p_bal < (p_fill > p_long ? p_fill : p_long)
                           ? p_bal
                           : (p_fill > p_long ? p_fill : p_long);
        if (np < 1) np = 1;
        // Wave fill: measured on B200 over four batch shapes, a grid whose
        // last wave of CTAs is about 55-70% full streamed best, and one that
        // spills a few CTAs into a new wave, or fills its last wave to 80% or
        // more, 2-16% worse.  So take, among half to twice that many
        // partitions (none under kMinPartitionPages, at least 1.4 waves, at
        // most kOneBatchSlots partials per row), the count whose last wave is
        // nearest 62% full, a partition more or less counting as 1%.  Batches
        // of so few units that no such grid exists (one or two long
        // sequences) take one partial wave instead, nearest 75% full.
        // Measured on B200 (8 kv heads), against the same rule without the
        // partials limit: 1 x 32768 tokens +45%, 2 x 32768 +20%, 1 and 2 x
        // 131072 with a shared prefix +24% and +7%, 4 and 6 x 131072 +3.1%
        // and +2.5%, 3 x 131072 with a prefix -1.1%.
        // Prefix CTAs per kv head and prefix partition, as counted below: W row
        // groups per CTA with a shared ring (at least W groups), else one each.
        const long long groups_est =
            cascade ? (static_cast<long long>(num_seqs) * (num_heads / num_kv_heads) + 15) / 16 : 0;
        const long long cta_groups_est = groups_est >= W ? (groups_est + W - 1) / W : groups_est;
        // Partition size for about n partitions of max_seq_len, evened out
        // over the pages each sequence splits (its own pages, after a shared
        // prefix) so that no partition is left much shorter than the others.
        const long long own = cascade ? pages_max - prefix : pages_max;
        auto part_pages = [&](long long n) {
            const long long q = (pages_max + n - 1) / n;
            const long long parts = (own + q - 1) / q;
            return parts > 0 ? (own + parts - 1) / parts : q;
        };
        auto grid_for = [&](long long n) {
            const long long q = part_pages(n);
            if (!cascade) return units * ((pages_max + q - 1) / q);
            return units * ((own + q - 1) / q) +
                   num_kv_heads * cta_groups_est * ((prefix + q - 1) / q);
        };
        auto row_slots = [&](long long n) {  // partials per query row
            const long long q = part_pages(n);
            if (!cascade) return (pages_max + q - 1) / q;
            return (own + q - 1) / q + (prefix + q - 1) / q;
        };
        long long best = np;
        double best_score = -1.0;
        for (long long n = np / 2 > 1 ? np / 2 : 1; n <= 2 * np; ++n) {
            if ((pages_max + n - 1) / n < kMinPartitionPages) break;
            const double w = static_cast<double>(grid_for(n)) / static_cast<double>(slots);
            if (w < 1.4) continue;
            const double f = w - static_cast<double>(static_cast<long long>(w));
            const double score = (f > 0.62 ? f - 0.62 : 0.62 - f) +
                                 0.01 * static_cast<double>(n > np ? n - np : np - n);
            if (row_slots(n) <= kOneBatchSlots && (best_score < 0.0 || score < best_score)) {
                best = n;
                best_score = score;
            }
        }
        if (best_score < 0.0) {
            // One partial wave of at least half the CTA slots (the grid grows
            // with n).
            double best1 = -1.0;
            for (long long n = 1;; ++n) {
                if (n > 1 && (pages_max + n - 1) / n < kMinPartitionPages) break;
                const double w = static_cast<double>(grid_for(n)) / static_cast<double>(slots);
                if (w >= 1.0 || row_slots(n) > kOneBatchSlots) break;
                if (w < 0.5) continue;
                const double score = w > 0.75 ? w - 0.75 : 0.75 - w;
                if (best1 < 0.0 || score < best1) {
                    best = n;
                    best1 = score;
                }
            }
            if (best1 < 0.0) {
                // A handful of units (fewer than 7 on 148 SMs): about
                // kFewUnitCtas CTAs (128 on 148 SMs), with up to
                // max(32, that / units) partials per row.  Measured on B200 with
                // 1, 2 and 4 units of 32768-131072 tokens: grids of 64-128 CTAs
                // streamed 1.5-2.6x faster than 432-632 CTAs of 108-432
                // partials per row, whose merge takes several batches of loads.
                long long few = static_cast<long long>(sms) * kFewUnitCtas / kFewUnitSms;
                if (few < 1) few = 1;
                const long long cap_slots = (few + units - 1) / units > kOneBatchSlots
                                                ? (few + units - 1) / units
                                                : kOneBatchSlots;
                for (long long n = 1;; ++n) {
                    if (n > 1 && (pages_max + n - 1) / n < kMinPartitionPages) break;
                    if (row_slots(n) > cap_slots) break;
                    best = n;
                }
            }
        }
        np = best;
        pp = part_pages(np);
    }
    if (pp < 1) pp = 1;
    long long P = pages_max > 0 ? (pages_max + pp - 1) / pp : 1;
    if (P <= 1) {
        P = 1;
        pp = pages_max > 0 ? pages_max : 1;
    }
    // Shared prefix: its pages are split like the rest; each sequence's own
    // pages (after the prefix) get their own partitions.
    long long p_pre = 0, groups = 0;
    if (cascade) {
        p_pre = (prefix + pp - 1) / pp;
        P = (pages_max - prefix + pp - 1) / pp;
        groups = (static_cast<long long>(num_seqs) * (num_heads / num_kv_heads) + 15) / 16;
    }
    // Split tail: with whole units in two or more waves, the units of the
    // last, partial wave (units mod CTA slots) are cut into kTailParts
    // partitions each, dispatched after every whole unit, so that the call
    // does not end on a few full-length units streaming alone.  Measured on
    // B200: in two or three waves, +2.4% to +4.0% on equal-length batches of
    // 1024 units and -0.2% to -0.35% when the last units are the short ones of
    // mixed lengths; from four waves up, +0.65% to +2.5% on batches of paired
    // pages (e4m3 pages of 16 tokens, bf16 pages of head size 64) and -1.1% to
    // +0.05% on the others, so there only paired pages are split.
    long long tail_units = 0;
    int tail_P = 0, tail_PP = 0;
    if (whole_units && !cascade && schedule == PA_SCHEDULE_AUTO && (units < 4 * slots || pair)) {
        const long long r = units % slots;
        // Enough partitions that the tail's CTAs about fill the slots, at least
        // kTailParts, at most kMaxTailParts, none under kMinPartitionPages.
        long long tp = r > 0 ? (slots + r - 1) / r : 0;
        if (tp < kTailParts) tp = kTailParts;
        if (tp > kMaxTailParts) tp = kMaxTailParts;
        while (tp > kTailParts && (pages_max + tp - 1) / tp < kMinPartitionPages) --tp;
        if (r > 0 && r <= kMergeCounts && (pages_max + tp - 1) / tp >= kMinPartitionPages) {
            tail_units = r;
            tail_P = static_cast<int>(tp);
            tail_PP = static_cast<int>((pages_max + tp - 1) / tp);
        }
    }
    // Short partitions: give each warp a buffer for every page it will read
    // (up to 4), so all copies are in flight after one block-table read.
    if (!(opts && opts->stages > 0)) {
        const long long per_warp = ((pp + (pair ? 1 : 0)) / (pair ? 2 : 1) + W - 1) / W;
        const size_t want = static_cast<size_t>(W) * per_warp * (stage + 8);
        if (per_warp > ns && per_warp <= kMaxShortStages && want <= kShortStagesSmem) {
            ns = static_cast<int>(per_warp);
            stage_area = static_cast<size_t>(W) * ns * stage;
            if (stage_area < mb) stage_area = mb;
            smem = stage_area + static_cast<size_t>(W) * ns * bar_bytes_per_buffer;
        }
    }
    if (pp > (1ll << 30) || P > (1ll << 30))
        return fail(PA_ERR_INVALID_ARG, "%s", "partition count out of range");

    size_t ws = PA_WORKSPACE_HEADER_BYTES;
    if (P > 1 || cascade || tail_P > 0) {
        // partials: per (seq, q head, partition), or per (tail unit, q head
        // of its group, tail partition)
        const size_t rows =
            tail_P > 0 ? static_cast<size_t>(tail_units) * (num_heads / num_kv_heads) * tail_P
                       : static_cast<size_t>(num_seqs) * num_heads * (P + p_pre);
        ws = kBodyOffset + rows * (static_cast<size_t>(head_size) + 2) * sizeof(float);
        ws = (ws + 255) & ~static_cast<size_t>(255);
    }
    pl->num_partitions = static_cast<int>(P);
    pl->partition_pages = static_cast<int>(pp);
    pl->stages = ns;
    pl->warps_per_cta = W;
    // Prefix units: a CTA per (kv head, prefix partition) and W row groups,
    // whose warps share one ring of its pages, when there are at least W
    // groups (measured on B200, 8 x 131072 tokens, 1024-block prefix: +0.8%
    // with 2 groups, +6.2% with 4, on two warps per CTA); with fewer, a CTA
    // per row group, its warps splitting the pages (a shared ring there would
    // leave warps idle: -1.0% with one group).
    const long long cta_groups = groups >= W ? (groups + W - 1) / W : groups;
    pl->grid_ctas = units * P + num_kv_heads * cta_groups * p_pre + tail_units * (tail_P - 1);
    pl->tail_units = tail_units;
    pl->tail_partitions = tail_P;
    pl->tail_partition_pages = tail_PP;
    // Longest first (ranked on the device) only when the grid takes more than
    // one wave of CTA slots: in one wave every CTA starts at once and the
    // order does not matter, and ranking would put the length loads ahead of
    // every block-table read.
    pl->longest_first =
        (num_seqs > 1 && num_seqs <= kMaxRankedSeqs && pl->grid_ctas > slots) ? 1 : 0;
    // Split partials are merged by the combine kernel (merging them in the
    // decode kernel, by each unit's last CTA, measured slower on B200: -1.7%
    // on the long-context workload, -3.9% on a 100 us call); the split tail's
    // are merged in the kernel.
    pl->combine = (P > 1 || cascade) ? 1 : 0;
    pl->smem_bytes = smem;
    pl->workspace_bytes = ws;
    pl->prefix_partitions = static_cast<int>(p_pre);
    pl->prefix_groups = static_cast<int>(groups);
    pl->balanced = 0;
    return PA_OK;
}

// Raise the kernel's dynamic shared-memory limit once per device.  `done` is
// owned by the caller's template instantiation, so every kernel variant keeps
// its own flags.
template <typename K>
cudaError_t ensure_smem(K kernel, std::atomic<int>* done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kMaxDevices;
    if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    // The opt-in limit covers static and dynamic shared memory together.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kMaxSmemPerCta - fa.sharedSizeBytes));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // do not leave the error for an unrelated later call
        return e;
    }
    if (cached) done[dev].store(1, std::memory_order_release);
    return e;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the kernel ahead of it in the stream drains, which hides the launch
// gap between back-to-back calls and between decode and combine.  Both
// kernels wait (griddepcontrol.wait) before touching memory, so stream order
// is kept for everything they read and write.
template <typename... Params>
cudaError_t launch_pdl(void (*kern)(Params...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t st, const Params&... p) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Forms with a CUDA-core variant for one query head per kv head: bf16 pages.
template <int D, int B, bool FP8, bool F8MMA>
constexpr bool has_scalar_form() {
    return !FP8 && !F8MMA;
}

template <int D, int B, bool FP8, int NH, bool F8MMA, bool SC = false>
cudaError_t launch_decode(const pa::DecodeParams& p, long long grid, size_t smem,
                          cudaStream_t st) {
    static std::atomic<int> done[kMaxDevices];
    constexpr int W = pa::decode_warps<D, B, FP8>();
    auto kern = pa::pa_decode_kernel<D, B, FP8, NH, W, F8MMA, SC>;
    if (smem > kMaxSmemPerCta - kStaticSmemReserve) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem(kern, done);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, static_cast<unsigned>(grid), W * 32, smem, st, p);
}

template <int D, int B, bool FP8, bool F8MMA>
cudaError_t launch_nh(const pa::DecodeParams& p, bool sc, long long grid, size_t smem,
                      cudaStream_t st) {
    if constexpr (has_scalar_form<D, B, FP8, F8MMA>()) {
        if (sc && p.G == 1 && p.prefix_pages == 0)
            return launch_decode<D, B, FP8, 1, F8MMA, true>(p, grid, smem, st);
    }
    // Shared-prefix units pack 16 query rows, so they need the 16-row form.
    return (p.G > 8 || p.prefix_pages > 0)
               ? launch_decode<D, B, FP8, 2, F8MMA>(p, grid, smem, st)
               : launch_decode<D, B, FP8, 1, F8MMA>(p, grid, smem, st);
}

template <int D, int B>
cudaError_t launch_dtype(const pa::DecodeParams& p, bool fp8, bool f8mma, bool sc,
                         long long grid, size_t smem, cudaStream_t st) {
    if (!fp8) return launch_nh<D, B, false, false>(p, sc, grid, smem, st);
    return f8mma ? launch_nh<D, B, true, true>(p, sc, grid, smem, st)
                 : launch_nh<D, B, true, false>(p, sc, grid, smem, st);
}

cudaError_t launch_any(const pa::DecodeParams& p, int D, int B, bool fp8, bool f8mma, bool sc,
                       long long grid, size_t smem, cudaStream_t st) {
    if (D == 64) return B == 16 ? launch_dtype<64, 16>(p, fp8, f8mma, sc, grid, smem, st)
                                : launch_dtype<64, 32>(p, fp8, f8mma, sc, grid, smem, st);
    return B == 16 ? launch_dtype<128, 16>(p, fp8, f8mma, sc, grid, smem, st)
                   : launch_dtype<128, 32>(p, fp8, f8mma, sc, grid, smem, st);
}

// The dynamic schedule's persistent grid: at most the CTAs that can be
// resident at once (the planner's slots, bounded by the occupancy of this
// kernel form), so that every warp runs from the start.
template <int D, int B, bool FP8, int NH, bool F8MMA, bool SC = false>
cudaError_t launch_dyn(const pa::DecodeParams& p, pa::DynParams t, long long grid, size_t smem,
                       cudaStream_t st) {
    static std::atomic<int> done[kMaxDevices];
    constexpr int W = pa::decode_warps<D, B, FP8>();
    auto kern = pa::pa_decode_dyn_kernel<D, B, FP8, NH, W, F8MMA, SC>;
    if (smem > kMaxSmemPerCta - kStaticSmemReserve) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem(kern, done);
    if (e != cudaSuccess) return e;
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, W * 32, smem);
    if (e != cudaSuccess) return e;
    if (device_sms(&sms) != 0) return cudaErrorInvalidDevice;
    const long long resident = static_cast<long long>(per_sm) * sms;
    if (resident > 0 && grid > resident) grid = resident;
    if (grid < 1) grid = 1;
    t.total_warps = static_cast<int>(grid * W);
    return launch_pdl(kern, static_cast<unsigned>(grid), W * 32, smem, st, p, t);
}

template <int D, int B, bool FP8, bool F8MMA>
cudaError_t launch_dyn_nh(const pa::DecodeParams& p, const pa::DynParams& t, bool sc,
                          long long grid, size_t smem, cudaStream_t st) {
    if constexpr (has_scalar_form<D, B, FP8, F8MMA>()) {
        if (sc && p.G == 1 && p.prefix_pages == 0)
            return launch_dyn<D, B, FP8, 1, F8MMA, true>(p, t, grid, smem, st);
    }
    return (p.G > 8 || p.prefix_pages > 0) ? launch_dyn<D, B, FP8, 2, F8MMA>(p, t, grid, smem, st)
                                           : launch_dyn<D, B, FP8, 1, F8MMA>(p, t, grid, smem, st);
}

template <int D, int B>
cudaError_t launch_dyn_dtype(const pa::DecodeParams& p, const pa::DynParams& t, bool fp8,
                             bool f8mma, bool sc, long long grid, size_t smem, cudaStream_t st) {
    if (!fp8) return launch_dyn_nh<D, B, false, false>(p, t, sc, grid, smem, st);
    return f8mma ? launch_dyn_nh<D, B, true, true>(p, t, sc, grid, smem, st)
                 : launch_dyn_nh<D, B, true, false>(p, t, sc, grid, smem, st);
}

cudaError_t launch_dyn_any(const pa::DecodeParams& p, const pa::DynParams& t, int D, int B,
                           bool fp8, bool f8mma, bool sc, long long grid, size_t smem,
                           cudaStream_t st) {
    if (D == 64) return B == 16 ? launch_dyn_dtype<64, 16>(p, t, fp8, f8mma, sc, grid, smem, st)
                                : launch_dyn_dtype<64, 32>(p, t, fp8, f8mma, sc, grid, smem, st);
    return B == 16 ? launch_dyn_dtype<128, 16>(p, t, fp8, f8mma, sc, grid, smem, st)
                   : launch_dyn_dtype<128, 32>(p, t, fp8, f8mma, sc, grid, smem, st);
}

cudaError_t launch_combine(const pa::CombineParams& c, int D, cudaStream_t st) {
    const long long rows = static_cast<long long>(c.S) * c.Hq;
    const unsigned grid = static_cast<unsigned>((rows + pa::kWarps - 1) / pa::kWarps);
    return D == 64 ? launch_pdl(pa::pa_combine_kernel<64>, grid, pa::kThreads, 0, st, c)
                   : launch_pdl(pa::pa_combine_kernel<128>, grid, pa::kThreads, 0, st, c);
}

// Every check pa_decode makes before planning, except on the workspace.
// *empty is set for a batch of no sequences (nothing to launch; its pointers
// are not looked at).
pa_status check_args(const void* out, const void* query, const void* key_cache,
                     const void* value_cache, int num_seqs, int num_heads, int num_kv_heads,
                     int head_size, float scale, const int32_t* block_tables,
                     int max_blocks_per_seq, const int32_t* seq_lens, int block_size,
                     int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                     const float* k_scale, const float* v_scale, const pa_options* opts,
                     bool* empty) {
    *empty = false;
    pa_status st = check_sizes(num_seqs, num_heads, num_kv_heads, head_size, block_size,
                               max_seq_len, kv_dtype);
    if (st != PA_OK) return st;
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "%s", "scale is not finite");
    if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID_ARG, "%s", "max_blocks_per_seq < 1");
    if (static_cast<long long>(max_seq_len) > static_cast<long long>(max_blocks_per_seq) * block_size)
        return fail(PA_ERR_INVALID_ARG, "%s", "max_seq_len > max_blocks_per_seq * block_size");
    if (num_blocks < 1) return fail(PA_ERR_INVALID_ARG, "%s", "num_blocks < 1");
    if (num_seqs == 0) {
        *empty = true;
        return PA_OK;
    }
    const struct {
        const void* p;
        size_t a;
        const char* name;
    } ptrs[] = {{out, 16, "out"},
                {query, 16, "query"},
                {key_cache, 16, "key_cache"},
                {value_cache, 16, "value_cache"},
                {block_tables, 4, "block_tables"},
                {seq_lens, 4, "seq_lens"}};
    for (const auto& q : ptrs) {
        if (!q.p) return fail(PA_ERR_INVALID_ARG, "%s is NULL", q.name);
        if (!aligned(q.p, q.a)) return fail(PA_ERR_INVALID_ARG, "%s is misaligned", q.name);
    }
    if (opts && opts->fp8_compute && kv_dtype != PA_KV_FP8_E4M3)
        return fail(PA_ERR_INVALID_ARG, "%s", "fp8_compute needs an e4m3 KV cache");
    if (opts && opts->alibi_slopes && !aligned(opts->alibi_slopes, 4))
        return fail(PA_ERR_INVALID_ARG, "%s", "alibi_slopes is misaligned");
    if (kv_dtype == PA_KV_FP8_E4M3) {
        if (!k_scale || !v_scale)
            return fail(PA_ERR_INVALID_ARG, "%s", "k_scale and v_scale are required for FP8");
        if (!aligned(k_scale, 4) || !aligned(v_scale, 4))
            return fail(PA_ERR_INVALID_ARG, "%s", "k_scale / v_scale misaligned");
    }
    return PA_OK;
}

// Scratch of pa_decode_noalloc: one fixed array per device, in the
// library's own device memory (no allocation at call time).
constexpr size_t kNoallocScratchBytes = PA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch in the calling thread's current
// context.  In host code the array's name is only a host-side stand-in, so
// the address is looked up with cudaGetSymbolAddress, once per context: a
// context is a separate address space (another context on the same device,
// or the new primary context after cudaDeviceReset, has its own copy of the
// array), so the cache is keyed by the context's unique id and not by the
// device number.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The current context's unique id (never reused within a process), or 0 when
// no context is current or the driver cannot say.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        (void)cudaGetLastError();
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

pa_status noalloc_scratch(void** out) {
    struct Entry {
        unsigned long long ctx;
        void* addr;
    };
    static std::mutex mu;
    static Entry cache[kMaxDevices];
    static int n_cached = 0;
    unsigned long long ctx = current_context_id();
    if (ctx != 0) {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < n_cached; ++i)
            if (cache[i].ctx == ctx) {
                *out = cache[i].addr;
                return PA_OK;
            }
    }
    // First call in this context (or the context is not known): look the
    // address up.  This binds the device's primary context to the thread when
    // none is current yet, and may load the library's device code into it.
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
        return fail(PA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    if (ctx == 0) ctx = current_context_id();
    if (ctx != 0) {
        std::lock_guard<std::mutex> lock(mu);
        int slot = -1;
        for (int i = 0; i < n_cached; ++i)
            if (cache[i].ctx == ctx) slot = i;
        if (slot < 0) {
            // A full table drops its oldest entry (contexts come and go).
            if (n_cached == kMaxDevices) {
                for (int i = 1; i < n_cached; ++i) cache[i - 1] = cache[i];
                --n_cached;
            }
            slot = n_cached++;
        }
        cache[slot] = Entry{ctx, p};
    }
    *out = p;
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_plan_decode(pa_plan* out, int num_seqs, int num_heads, int num_kv_heads,
                         int head_size, int block_size, int max_seq_len, pa_kv_dtype kv_dtype,
                         const pa_options* opts) {
    g_detail[0] = 0;
    if (!out) return fail(PA_ERR_INVALID_ARG, "%s", "plan is NULL");
    return plan(out, num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len,
                kv_dtype, opts);
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                int block_size, int max_seq_len, pa_kv_dtype kv_dtype,
                                const pa_options* opts) {
    g_detail[0] = 0;
    pa_plan pl;
    if (plan(&pl, num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len, kv_dtype,
             opts) != PA_OK)
        return 0;
    return pl.workspace_bytes;
}

pa_status pa_decode_ex(void* out, const void* query, const void* key_cache,
                       const void* value_cache, int num_seqs, int num_heads, int num_kv_heads,
                       int head_size, float scale, const int32_t* block_tables,
                       int max_blocks_per_seq, const int32_t* seq_lens, int block_size,
                       int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                       const float* k_scale, const float* v_scale, void* workspace,
                       size_t workspace_bytes, void* stream, const pa_options* opts) {
    g_detail[0] = 0;
    bool empty = false;
    pa_status st = check_args(out, query, key_cache, value_cache, num_seqs, num_heads,
                              num_kv_heads, head_size, scale, block_tables, max_blocks_per_seq,
                              seq_lens, block_size, max_seq_len, num_blocks, kv_dtype, k_scale,
                              v_scale, opts, &empty);
    if (st != PA_OK || empty) return st;
    if (!workspace) return fail(PA_ERR_INVALID_ARG, "%s", "workspace is NULL");
    if (!aligned(workspace, 16)) return fail(PA_ERR_INVALID_ARG, "%s", "workspace is misaligned");
    pa_plan pl;
    st = plan(&pl, num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len, kv_dtype,
              opts);
    if (st != PA_OK) return st;
    if (workspace_bytes < pl.workspace_bytes)
        return fail(PA_ERR_WORKSPACE_TOO_SMALL, "%s", "workspace_bytes < pa_decode_workspace_size");
    if (pl.grid_ctas > 0x7fffffffll) return fail(PA_ERR_INVALID_ARG, "%s", "grid too large");

    pa::DecodeParams p;
    std::memset(&p, 0, sizeof p);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.q = static_cast<const uint16_t*>(query);
    p.kc = static_cast<const uint8_t*>(key_cache);
    p.vc = static_cast<const uint8_t*>(value_cache);
    p.bt = block_tables;
    p.seq_lens = seq_lens;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.status = reinterpret_cast<uint32_t*>(ws);
    const int p_total = pl.num_partitions + pl.prefix_partitions;
    size_t rows = static_cast<size_t>(num_seqs) * num_heads * p_total;
    float* part = reinterpret_cast<float*>(ws + kBodyOffset);
    if (pl.balanced) {
        // [header][per-sequence page scan, S + 2 ints][slots: 2 per CTA, G rows each]
        p.br_scan = reinterpret_cast<int*>(ws + kBodyOffset);
        const size_t scan_bytes =
            ((static_cast<size_t>(num_seqs) + 2) * sizeof(int) + 255) & ~static_cast<size_t>(255);
        part = reinterpret_cast<float*>(ws + kBodyOffset + scan_bytes);
        rows = 2 * static_cast<size_t>(pl.grid_ctas) * (num_heads / num_kv_heads);
    }
    if (pl.tail_partitions > 0)
        rows = static_cast<size_t>(pl.tail_units) * (num_heads / num_kv_heads) * pl.tail_partitions;
    p.ws_o = part;
    p.ws_m = part + rows * head_size;
    p.ws_l = p.ws_m + rows;
    p.n_full = static_cast<long long>(num_seqs) * num_kv_heads - pl.tail_units;
    p.tail_P = pl.tail_partitions;
    p.tail_PP = pl.tail_partition_pages;
    p.merge_cnt = pl.tail_partitions > 0
                      ? reinterpret_cast<unsigned int*>(ws + PA_WORKSPACE_HEADER_BYTES)
                      : nullptr;
    p.S = num_seqs;
    p.Hq = num_heads;
    p.Hk = num_kv_heads;
    p.G = num_heads / num_kv_heads;
    p.max_blocks = max_blocks_per_seq;
    p.P = pl.num_partitions;
    p.PP = pl.partition_pages;
    p.stages = pl.stages;
    p.num_blocks = num_blocks;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.prefix_pages = pl.prefix_partitions > 0 ? opts->shared_prefix_blocks : 0;
    p.prefix_parts = pl.prefix_partitions;
    p.prefix_groups = pl.prefix_groups;
    p.prefix_shared = pl.prefix_groups >= pl.warps_per_cta ? 1 : 0;
    p.prefix_cta_groups = p.prefix_shared
                              ? (pl.prefix_groups + pl.warps_per_cta - 1) / pl.warps_per_cta
                              : pl.prefix_groups;
    p.prefix_units =
        static_cast<long long>(num_kv_heads) * p.prefix_cta_groups * pl.prefix_partitions;
    p.P_total = p_total;
    p.alibi = opts ? opts->alibi_slopes : nullptr;
    p.longest_first = pl.longest_first;
    p.balanced = pl.balanced;
    p.stall_tx_bytes = 0;
    p.wait_limit_ns = kWaitLimitNs;
    if (opts && opts->test_stall_copies) {
        p.stall_tx_bytes = 16;
        p.wait_limit_ns = kTestWaitLimitNs;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool f8mma = opts && opts->fp8_compute && kv_dtype == PA_KV_FP8_E4M3;
    const bool sc = opts && opts->mha_cuda_cores;
    if (pl.dynamic) {
        // [header: status, ..., generation / unit cursor / warps finished at
        //  byte 64][unit counters, 16 bytes per unit][partials: rows x slots]
        const bool pair =
            block_size == 16 && (kv_dtype == PA_KV_FP8_E4M3 || head_size == 64);
        const int npg = pair ? 2 : 1;
        pa::DynParams t;
        std::memset(&t, 0, sizeof t);
        t.units_pre = num_kv_heads * pl.prefix_groups;
        t.units = t.units_pre + num_seqs * num_kv_heads;
        t.owners = pl.dynamic;
        t.k_pre = pl.prefix_partitions;
        t.k_own = pl.num_partitions;
        t.k_total = t.k_pre + t.k_own;
        t.step_min = 4 * npg;
        t.step_max = 32 * npg;
        t.probe_rounds = (t.units + 31) / 32 < 8 ? (t.units + 31) / 32 : 8;
        t.hdr = reinterpret_cast<unsigned int*>(ws + 4 * pa::kDynHeaderWord);
        t.uw = reinterpret_cast<unsigned long long*>(ws + kBodyOffset);
        const size_t uw_bytes =
            (static_cast<size_t>(t.units) * 16 + 255) & ~static_cast<size_t>(255);
        float* dpart = reinterpret_cast<float*>(ws + kBodyOffset + uw_bytes);
        const size_t drows = static_cast<size_t>(num_seqs) * num_heads * t.k_total;
        p.ws_o = dpart;
        p.ws_m = dpart + drows * head_size;
        p.ws_l = p.ws_m + drows;
        cudaError_t e = launch_dyn_any(p, t, head_size, block_size, kv_dtype == PA_KV_FP8_E4M3,
                                       f8mma, sc, pl.grid_ctas, pl.smem_bytes, s);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
        pa::CombineParams c;
        std::memset(&c, 0, sizeof c);
        c.out = p.out;
        c.ws_o = p.ws_o;
        c.ws_m = p.ws_m;
        c.ws_l = p.ws_l;
        c.seq_lens = seq_lens;
        c.S = num_seqs;
        c.Hq = num_heads;
        c.max_blocks = max_blocks_per_seq;
        c.B = block_size;
        c.prefix_pages = p.prefix_pages;
        c.Hk = num_kv_heads;
        c.G = num_heads / num_kv_heads;
        c.dynamic = 1;
        c.dyn_units_pre = t.units_pre;
        c.dyn_owners = t.owners;
        c.dyn_k_pre = t.k_pre;
        c.dyn_k_own = t.k_own;
        c.dyn_k_total = t.k_total;
        c.dyn_hdr = t.hdr;
        c.dyn_uw = t.uw;
        e = launch_combine(c, head_size, s);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
        return PA_OK;
    }
    cudaError_t e = launch_any(p, head_size, block_size, kv_dtype == PA_KV_FP8_E4M3, f8mma, sc,
                               pl.grid_ctas, pl.smem_bytes, s);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    if (pl.combine) {
        pa::CombineParams c;
        std::memset(&c, 0, sizeof c);
        c.out = p.out;
        c.ws_o = p.ws_o;
        c.ws_m = p.ws_m;
        c.ws_l = p.ws_l;
        c.seq_lens = seq_lens;
        c.S = num_seqs;
        c.Hq = num_heads;
        c.P = pl.num_partitions;
        c.PP = pl.partition_pages;
        c.max_blocks = max_blocks_per_seq;
        c.B = block_size;
        c.prefix_pages = p.prefix_pages;
        c.prefix_parts = p.prefix_parts;
        c.P_total = p.P_total;
        c.balanced = pl.balanced;
        c.Hk = num_kv_heads;
        c.G = num_heads / num_kv_heads;
        c.br_scan = p.br_scan;
        e = launch_combine(c, head_size, s);
        if (e != cudaSuccess) return fail(PA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
    }
    return PA_OK;
}

pa_status pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                    int num_seqs, int num_heads, int num_kv_heads, int head_size, float scale,
                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
                    int block_size, int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                    const float* k_scale, const float* v_scale, void* workspace,
                    size_t workspace_bytes, void* stream) {
    return pa_decode_ex(out, query, key_cache, value_cache, num_seqs, num_heads, num_kv_heads,
                        head_size, scale, block_tables, max_blocks_per_seq, seq_lens, block_size,
                        max_seq_len, num_blocks, kv_dtype, k_scale, v_scale, workspace,
                        workspace_bytes, stream, nullptr);
}

pa_status pa_decode_noalloc(void* out, const void* query, const void* key_cache,
                            const void* value_cache, int num_seqs, int num_heads, int num_kv_heads,
                            int head_size, float scale, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* seq_lens, int block_size,
                            int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                            const float* k_scale, const float* v_scale, void* stream) {
    g_detail[0] = 0;
    // The argument checks of pa_decode come first, so a bad argument is
    // reported as such whatever the problem's size.
    bool empty = false;
    pa_status st = check_args(out, query, key_cache, value_cache, num_seqs, num_heads,
                              num_kv_heads, head_size, scale, block_tables, max_blocks_per_seq,
                              seq_lens, block_size, max_seq_len, num_blocks, kv_dtype, k_scale,
                              v_scale, nullptr, &empty);
    if (st != PA_OK || empty) return st;
    pa_plan pl;
    st = plan(&pl, num_seqs, num_heads, num_kv_heads, head_size, block_size, max_seq_len, kv_dtype,
              nullptr);
    if (st != PA_OK) return st;
    if (pl.workspace_bytes > kNoallocScratchBytes) {
        std::snprintf(g_detail, sizeof g_detail,
                      "this problem needs %zu bytes of scratch; the built-in scratch holds %zu",
                      pl.workspace_bytes, kNoallocScratchBytes);
        return PA_ERR_WORKSPACE_TOO_SMALL;
    }
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != PA_OK) return st;
    return pa_decode_ex(out, query, key_cache, value_cache, num_seqs, num_heads, num_kv_heads,
                        head_size, scale, block_tables, max_blocks_per_seq, seq_lens, block_size,
                        max_seq_len, num_blocks, kv_dtype, k_scale, v_scale, scratch,
                        kNoallocScratchBytes, stream, nullptr);
}

pa_status pa_read_device_status(void* workspace, uint32_t* flags, int clear, void* stream) {
    g_detail[0] = 0;
    if (!workspace || !flags) return fail(PA_ERR_INVALID_ARG, "%s", "workspace or flags is NULL");
    if (!aligned(workspace, 16)) return fail(PA_ERR_INVALID_ARG, "%s", "workspace is misaligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear) e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    return PA_OK;
}

const char* pa_status_string(pa_status status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: unsupported shape or dtype";
        case PA_ERR_WORKSPACE_TOO_SMALL: return "PA_ERR_WORKSPACE_TOO_SMALL: workspace too small";
        case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime error";
        case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS: no free block or row full";
    }
    return "unknown pa_status";
}

const char* pa_last_error_detail(void) { return g_detail; }

int pa_version(void) { return kVersion; }

}  // extern "C"
