// Soft collision scoring: score(n) = vnorm(n) * sum_l T_l[id_l(n)] for every
// live key of every unit, where T_l is the unit's summed soft-assignment
// table of hash table l.
//
// Method: "Resumen Técnico: SOCKET ..." (gist.science/es/paper/2602.06283),
// "Mecanismo Central: LSH Suave" step 3 "Puntuación"; "SOCKET: SOft Collision
// Kernel EsTimator for Sparse Attention" (gist.science/de/paper/2602.06283),
// "Bewertung": the probability mass the query puts on the key's own bucket,
// aggregated over the L tables and weighted by the key's value norm.  The
// pages implement this step as "a custom CUDA scoring kernel"
// ("Contribuciones Clave" 2 / "Hauptbeiträge").
//
// B200 design.  The step streams the key's id row (one byte per table) and
// its fp32 norm from HBM and performs L random lookups into 2^P-entry tables.
// The lookups go to shared memory, conflict-free for any ids, without
// replicating the tables:
//   * every key has an id row rotated by the key: slot s of block c (32
//     tables) of key n holds the id of table 32c + (s + n) mod 32; rows are
//     stored in chunks of 32 keys, piece-major, so the 32 lanes' 16-byte loads
//     of one piece form one contiguous 512-byte warp load;
//   * a block's tables sit in a 64 KB region as float[bucket][64 columns],
//     column j holding table 32c + j mod 32 (written in that form by the
//     soft-table kernel and copied in with one bulk copy);
//   * lane j of a warp scores key 32m + j and, in round r, reads column
//     j + r of the row of its id for slot r -- table 32c + (j + r) mod 32, the
//     table slot r holds for that key -- so the 32 lanes of every lookup hit
//     32 distinct banks.
// A region starts at a 64 KB-aligned shared address, so one byte-permute of
// the packed id word (id into byte 1, lane column in byte 0) gives the row
// address and the round's column is the load's immediate offset: a lookup is
// one PRMT, one LDS and half a packed two-key FADD.  Each warp streams its batches (KEYS
// consecutive 32-key chunks of id pieces and norms, one bulk copy each) into
// its own ring of shared-memory stages on mbarriers, and reads them back with
// conflict-free 16-byte loads; ids and norms stream through L2 with an
// evict-first policy and the scores are stored evict-last, so top-k reads
// them from L2.  The grid is persistent (one CTA per SM) and splits the
// flattened (kv unit, 32-key chunk) range evenly; a CTA stages the tables of
// each unit it touches (two units at once when a unit needs one region).
// When every query head selects its own keys, the `share` units of a kv
// unit (one per head) read the same ids and norms: the grid is then groups
// of `share` CTAs, CTA h of a group scoring head h over the group's chunk
// range, so the group's CTAs stream the same id chunks at about the same
// time and all but the first read of each chunk is served from L2.
#include "common.cuh"
#include "internal.h"
#include "socket_attn.h"

namespace socket_attn {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kRegionBytes = 1u << 16;  // [256 buckets][64 columns] floats
constexpr int kMaxRegions = 2;
constexpr int kHistBins = kScoreHistBins;  // unit histogram of score bit patterns >> kHistShift
constexpr int kHistShift = kScoreHistShift;
// The regions sit at 64 KB-aligned shared addresses inside the dynamic
// allocation; the histogram and the copy rings use the space around them.
constexpr int kSmemBytes = 226 * 1024;
constexpr uint32_t kMaxPolls = 1u << 22;


__device__ __forceinline__ float lds_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// (a, b) += (x, y) as one packed float32x2 add (round to nearest), the same
// two float32 additions as a += x and b += y.
__device__ __forceinline__ void add_f32x2(float& a, float& b, float x, float y)
{
    asm("{.reg .b64 ra, rb;\n\t"
        "mov.b64 ra, {%0, %1};\n\t"
        "mov.b64 rb, {%2, %3};\n\t"
        "add.rn.f32x2 ra, ra, rb;\n\t"
        "mov.b64 {%0, %1}, ra;}"
        : "+f"(a), "+f"(b)
        : "f"(x), "f"(y));
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

struct ScoreArgs {
    const float* tables;  // [U][nblk][NB][64] expanded soft tables
    const uint8_t* ids;   // [U / share][Ncap][32 nblk] rotated id rows
    const float* vnorm;   // [U / share][Ncap]
    float* scores;        // [U][Ncap]
    uint32_t* unit_hist;
    uint32_t* err_word;
    int share;            // units per kv unit (CTAs per group)
    int nblk;             // 32-table blocks of L
    int blk0;             // first block of this launch
    int NB;
    int first, last;      // first / last launch of the step (partial sums between)
    int64_t Ncap, N;
    int64_t chunks_per_unit, total_chunks, chunks_per_cta;  // over kv units; per group of CTAs
    int64_t fresh_chunk;  // chunks from here on get ids in this step: not fetched before the wait
    uint32_t max_polls;   // polls before a wait for data gives up (draining waits use kMaxPolls)
};

// NBLK: 32-table blocks scored by this launch (1 or 2); REGIONS: 64 KB table
// regions in shared memory (REGIONS / (NBLK HPC) segments staged at once);
// KEYS: 32-key chunks per warp per batch; NS: batches in a warp's copy ring;
// FIRST / LAST: whether this launch starts / finishes the sum (launches in
// between pass partial sums through the score buffer); HPC: units (query
// heads, when every head selects its own keys) scored by one CTA from the
// same id rows -- each id row's loads and byte permutes serve all of them,
// and two heads' sums advance in one packed add.
template <int NBLK, int REGIONS, int KEYS, int NS, bool FIRST, bool LAST, int HPC = 1>
__global__ __launch_bounds__(kThreads, 1) void score_kernel(const ScoreArgs a)
{
    static_assert(REGIONS >= NBLK * HPC && REGIONS <= kMaxRegions, "a segment's blocks fit the regions");
    static_assert(HPC == 1 || (HPC == 2 && NBLK == 1 && FIRST && LAST), "two units per CTA: one launch, L <= 32");
    constexpr int V = 2 * NBLK;                            // 16-byte id pieces per key
    constexpr int kSlots = REGIONS / (NBLK * HPC);         // segments staged at once
    constexpr uint32_t kChunkIds = 1024u * NBLK;           // id bytes of a chunk in this launch
    constexpr uint32_t kChunkBytes = kChunkIds + (LAST ? 128u : 0u);  // + the chunk's norms
    constexpr uint32_t kStageBytes = KEYS * kChunkBytes;
    constexpr uint32_t kRingBytes = NS * kStageBytes;
    constexpr uint32_t kHistBytes = LAST ? HPC * kHistBins * 4u : 0u;
    extern __shared__ __align__(1024) char smem[];
    __shared__ __align__(8) uint64_t bar[kSlots];
    __shared__ __align__(8) uint64_t ring_bar[kWarps][NS];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t region0 = (sbase + kRegionBytes - 1) & ~(kRegionBytes - 1);
    char* region0_ptr = smem + (region0 - sbase);

    // The histogram and the warps' copy rings fill the space below the two
    // table regions, then the space above them.
    uint32_t lo = sbase, hi = region0 + REGIONS * kRegionBytes;
    const uint32_t lo_end = region0, hi_end = sbase + kSmemBytes;
    auto place = [&](uint32_t bytes) -> uint32_t {
        if (lo + bytes <= lo_end) { lo += bytes; return lo - bytes; }
        if (hi + bytes <= hi_end) { hi += bytes; return hi - bytes; }
        return 0u;
    };
    const uint32_t hist_s = LAST ? place(kHistBytes) : sbase;
    uint32_t ring_s = 0;
    bool fits = hist_s != 0u;
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t r = place(kRingBytes);
        fits = fits && r != 0u;
        if (w == warp) ring_s = r;
    }
    if (!fits) {  // cannot happen with the sizes launched; reported, not trapped
        if (tid == 0) atomicOr(a.err_word, SOCKET_DEVERR_TABLE_TIMEOUT);
        return;
    }
    uint32_t* shist = reinterpret_cast<uint32_t*>(smem + (hist_s - sbase));
    char* ring = smem + (ring_s - sbase);

    const unsigned cpg = (unsigned)(a.share / HPC);        // CTAs per group
    const int h = (int)(blockIdx.x % cpg) * HPC;           // this CTA's first unit within each kv unit
    const int64_t c0 = (int64_t)(blockIdx.x / cpg) * a.chunks_per_cta;
    const int64_t c1 = min64(a.total_chunks, c0 + a.chunks_per_cta);
    if (c0 >= c1) return;
    const int cpu = (int)a.chunks_per_unit;
    const int64_t u_first = c0 / cpu;  // first kv unit
    const int nseg = (int)((c1 - 1) / cpu - u_first + 1);
    const int Lr = 32 * a.nblk;  // id row bytes
    const int N = (int)a.N;
    const uint32_t region_bytes = (uint32_t)a.NB * 256u;

    // Let the next kernel on the stream get its CTAs queued behind this grid.
    pdl_launch_dependents();
    if (LAST)
        for (int b = tid; b < HPC * kHistBins; b += kThreads) shist[b] = 0;
    if (tid == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(&bar[s], 1);
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < NS; ++s) mbar_init(&ring_bar[w][s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();

    // Bulk copy of segment k's table blocks into its slot's regions (unit
    // h + hh's blocks at regions (s HPC + hh) NBLK + bl).
    auto issue_tables = [&](int k) {
        const int s = k % kSlots;
        mbar_arrive_expect_tx(&bar[s], HPC * NBLK * region_bytes);
        for (int hh = 0; hh < HPC; ++hh) {
            const int64_t u = (u_first + k) * a.share + h + hh;
            for (int bl = 0; bl < NBLK; ++bl) {
                const char* src = reinterpret_cast<const char*>(a.tables) +
                                  ((u * a.nblk + a.blk0 + bl) * (int64_t)region_bytes);
                char* dst = region0_ptr + ((s * HPC + hh) * NBLK + bl) * kRegionBytes;
                for (uint32_t off = 0; off < region_bytes; off += 16384u)
                    bulk_copy_g2s(dst + off, src + off, min(16384u, region_bytes - off), &bar[s]);
            }
        }
    };

    // Ids and norms stream through L2 once; the scores stay there for top-k.
    const uint64_t pol_stream = l2_policy_evict_first(), pol_keep = l2_policy_evict_last();
    uint32_t seq = 0;      // batches this warp has taken from its ring so far
    bool failed = false;   // a bounded wait of this warp expired
    for (int k = 0; k < nseg; ++k) {
        const int64_t ukv = u_first + k;
        const int64_t u = ukv * a.share + h;
        const int cbeg = (int)(max64(c0, ukv * cpu) - ukv * cpu);
        const int nch = (int)(min64(c1, (ukv + 1) * cpu) - ukv * cpu) - cbeg;
        const int slot = k % kSlots;
        // Batch b of this warp holds the KEYS consecutive chunks starting at
        // cbeg + (warp + kWarps b) KEYS (the last group of the segment may be
        // shorter); m = KEYS b + j indexes its chunks.
        const int ngroups = (nch + KEYS - 1) / KEYS;
        const int nbatch = ngroups > warp ? (ngroups - warp + kWarps - 1) / kWarps : 0;
        auto chunk_at = [&](int m) { return cbeg + (warp + kWarps * (m / KEYS)) * KEYS + (m % KEYS); };
        const int cend = cbeg + nch;
        const uint8_t* idu = a.ids + ukv * a.Ncap * Lr;
        const float* vu = a.vnorm + ukv * a.Ncap;
        float* su = a.scores + u * a.Ncap;

        // Lane 0: copy batch b's chunks (this launch's id pieces and, in the
        // last launch, the norms) into ring stage (seq + b) % NS, laid out as
        // [KEYS chunks of ids][KEYS x 32 norms].  When the launch covers the
        // whole id row, the chunks' ids are one contiguous run.  The unit's
        // last chunk may run past N (rows below Ncap, never scored).
        auto issue = [&](int b) {
            const uint32_t st = (seq + b) % NS;
            char* dst = ring + st * kStageBytes;
            const int c0 = chunk_at(b * KEYS);
            const int nv = min(KEYS, cend - c0);
            mbar_arrive_expect_tx(&ring_bar[warp][st], (uint32_t)nv * kChunkBytes);
            if (NBLK == a.nblk) {
                bulk_copy_g2s_hint(dst, idu + (int64_t)c0 * 32 * Lr, (uint32_t)nv * kChunkIds, &ring_bar[warp][st],
                                   pol_stream);
            } else {
                for (int j = 0; j < nv; ++j)
                    bulk_copy_g2s_hint(dst + j * kChunkIds, idu + (int64_t)(c0 + j) * 32 * Lr + (2 * a.blk0) * 512,
                                       kChunkIds, &ring_bar[warp][st], pol_stream);
            }
            if (LAST)
                bulk_copy_g2s_hint(dst + KEYS * kChunkIds, vu + (int64_t)c0 * 32, (uint32_t)nv * 128u,
                                   &ring_bar[warp][st], pol_stream);
        };
        // The stages were read in the previous segment: fence every lane's reads.
        fence_proxy_async_shared();
        __syncwarp();
        // The first segment's first batches are fetched before the wait below,
        // unless they reach a chunk whose ids the soft-table kernel writes in
        // this step (keys hashed on append).
        const int nfirst = min(NS, nbatch);
        const bool early = k > 0 || nfirst == 0 || chunk_at(nfirst * KEYS - 1) < a.fresh_chunk;
        int issued = 0;  // batches of this segment copied so far (warp-uniform)
        if (!failed && early) {
            if (lane == 0)
                for (int b = 0; b < nfirst; ++b) issue(b);
            issued = nfirst;
        }
        if (k == 0) {
            // The soft tables (and, after the first launch, the partial sums)
            // come from the previous kernel on the stream.
            pdl_wait();
            if (!failed && !early) {
                if (lane == 0)
                    for (int b = 0; b < nfirst; ++b) issue(b);
                issued = nfirst;
            }
            if (tid == 0)
                for (int kk = 0; kk < min(kSlots, nseg); ++kk) issue_tables(kk);
        }
        // Waits give up after a bounded number of polls; a warp gives up as a
        // whole so it never splits around __syncwarp.
        const bool tables_ok = mbar_wait_bounded(&bar[slot], (uint32_t)((k / kSlots) & 1), a.max_polls);
        if (__any_sync(kFullMask, !tables_ok)) {
            if (lane == 0) atomicOr(a.err_word, SOCKET_DEVERR_TABLE_TIMEOUT);
            mbar_wait_bounded(&bar[slot], (uint32_t)((k / kSlots) & 1), kMaxPolls);
            failed = true;
        }

        int b = 0;
        for (; b < nbatch && !failed; ++b) {
            const uint32_t st = (seq + b) % NS;
            const bool ids_ok = mbar_wait_bounded(&ring_bar[warp][st], ((seq + b) / NS) & 1u, a.max_polls);
            if (__any_sync(kFullMask, !ids_ok)) {
                if (lane == 0) atomicOr(a.err_word, SOCKET_DEVERR_TABLE_TIMEOUT);
                failed = true;
                break;
            }
            const uint32_t sa = ring_s + st * kStageBytes;
            uint4 v[KEYS][V];
            float vn[KEYS];
#pragma unroll
            for (int j = 0; j < KEYS; ++j) {
#pragma unroll
                for (int i = 0; i < V; ++i) v[j][i] = lds_u4(sa + j * kChunkIds + i * 512 + lane * 16);
                vn[j] = LAST ? lds_f32(sa + KEYS * kChunkIds + j * 128 + lane * 4) : 0.0f;
            }
            // Every lane's reads of this stage precede the next copy into it.
            fence_proxy_async_shared();
            __syncwarp();
            if (b + NS < nbatch) {
                if (lane == 0) issue(b + NS);
                issued = b + NS + 1;
            }
            float acc[KEYS][HPC];
#pragma unroll
            for (int j = 0; j < KEYS; ++j)
#pragma unroll
                for (int hh = 0; hh < HPC; ++hh)
                    acc[j][hh] = FIRST ? 0.0f
                                       : __ldcg(su + hh * a.Ncap +
                                                min(min(chunk_at(b * KEYS + j), cend - 1) * 32 + lane, N - 1));
#pragma unroll
            for (int bl = 0; bl < NBLK; ++bl) {
                // Unit h + hh's block bl sits 64 KB x hh (NBLK) above unit h's.
                const uint32_t base =
                    region0 + (uint32_t)(slot * HPC * NBLK + bl) * kRegionBytes + ((uint32_t)lane << 2);
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    const int q = bl * 32 + r;  // id byte within this launch's part of the row
                    // byte 1 <- the id (row), bytes 0, 2, 3 <- region and lane column
                    auto row = [&](int j) {
                        return __byte_perm(base, word_of(v[j][q >> 4], (q >> 2) & 3), 0x3240u | ((q & 3) << 4));
                    };
                    if constexpr (HPC == 2) {
                        // the two units' sums of a key advance in one packed float32x2 add
#pragma unroll
                        for (int j = 0; j < KEYS; ++j) {
                            const uint32_t rw = row(j);
                            add_f32x2(acc[j][0], acc[j][1], lds_f32(rw + 4u * r),
                                      lds_f32(rw + (uint32_t)(NBLK * kRegionBytes) + 4u * r));
                        }
                    } else if constexpr (KEYS % 2 == 0) {
                        // two keys' sums advance in one packed float32x2 add
#pragma unroll
                        for (int j = 0; j < KEYS; j += 2)
                            add_f32x2(acc[j][0], acc[j + 1][0], lds_f32(row(j) + 4u * r),
                                      lds_f32(row(j + 1) + 4u * r));
                    } else {
#pragma unroll
                        for (int j = 0; j < KEYS; ++j) acc[j][0] += lds_f32(row(j) + 4u * r);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < KEYS; ++j) {
                const int c = chunk_at(b * KEYS + j);
                const int n = c * 32 + lane;
                if (c < cend && n < N) {
#pragma unroll
                    for (int hh = 0; hh < HPC; ++hh) {
                        const float sc = LAST ? acc[j][hh] * vn[j] : acc[j][hh];
                        st_global_hint(su + hh * a.Ncap + n, sc, pol_keep);
                        if (LAST)
                            atomicAdd(shist + hh * kHistBins +
                                          min(__float_as_uint(sc) >> kHistShift, (uint32_t)(kHistBins - 1)),
                                      1u);
                    }
                }
            }
        }
        if (failed) {
            // Let this warp's copies in flight land before anything moves on.
            for (int bb = b; bb < issued; ++bb)
                mbar_wait_bounded(&ring_bar[warp][(seq + bb) % NS], ((seq + bb) / NS) & 1u, kMaxPolls);
        }
        seq += nbatch;

        if (LAST) {
            // The units' score histograms.
            __syncthreads();
            uint32_t* gh = a.unit_hist + u * kHistBins;  // units u .. u + HPC - 1 are adjacent
            for (int bn = tid; bn < HPC * kHistBins; bn += kThreads) {
                const uint32_t c = shist[bn];
                if (c) {
                    atomicAdd(gh + bn, c);
                    shist[bn] = 0;
                }
            }
        }
        if (k + kSlots < nseg) {
            __syncthreads();  // every warp is done with this slot's regions
            if (tid == 0) issue_tables(k + kSlots);
        } else if (LAST) {
            __syncthreads();  // histogram cleared before the next segment counts
        }
    }
}

template <int NBLK, int REGIONS, int KEYS, int NS, bool FIRST, bool LAST, int HPC = 1>
cudaError_t launch_one(const ScoreArgs& args, int grid, cudaStream_t stream)
{
    auto kern = score_kernel<NBLK, REGIONS, KEYS, NS, FIRST, LAST, HPC>;
    cudaError_t e = set_smem_limit_once((const void*)kern, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

int ids_row_bytes(int L) { return 32 * ((L + 31) / 32); }

cudaError_t launch_score(const float* tables, const uint8_t* ids, const float* vnorm, const DecodeShape& s,
                         int64_t fresh_chunk, float* scores, uint32_t* unit_hist, uint32_t* err_word,
                         cudaStream_t stream)
{
    ScoreArgs a;
    a.tables = tables;
    a.ids = ids;
    a.vnorm = vnorm;
    a.scores = scores;
    a.unit_hist = unit_hist;
    a.err_word = err_word;
    a.nblk = (s.L + 31) / 32;
    a.NB = s.NB;
    a.Ncap = s.Ncap;
    a.N = s.N;
    a.share = s.share;
    a.fresh_chunk = fresh_chunk;
    a.max_polls = wait_poll_limit();
    a.chunks_per_unit = (s.N + 31) / 32;
    a.total_chunks = (s.U / s.share) * a.chunks_per_unit;
    // When every query head selects its own keys and L <= 32, a CTA scores two
    // heads of a kv unit from one stream of its ids.
    const int hpc = (s.share % 2 == 0 && a.nblk == 1) ? 2 : 1;
    const int cpg = s.share / hpc;  // CTAs per group
    // At least one chunk per warp per CTA; at most one CTA per SM; groups of
    // `cpg` CTAs.
    const int64_t want = (a.total_chunks + kWarps - 1) / kWarps;
    const int64_t groups = max64(1, min64(device_num_sms() / cpg, want));
    const int grid = (int)(groups * cpg);
    a.chunks_per_cta = (a.total_chunks + groups - 1) / groups;
    // Blocks two at a time (two 64 KB regions); partial sums pass through
    // the score buffer between launches when L > 64.
    for (int b0 = 0; b0 < a.nblk; b0 += kMaxRegions) {
        const int nb = min(kMaxRegions, a.nblk - b0);
        a.blk0 = b0;
        a.first = b0 == 0;
        a.last = b0 + nb == a.nblk;
        cudaError_t e;
        if (nb == 1 && hpc == 2)
            e = launch_one<1, 2, 1, 3, true, true, 2>(a, grid, stream);  // one launch: nblk == 1
        else if (nb == 1)
            e = a.first ? launch_one<1, 2, 2, 2, true, true>(a, grid, stream)
                        : launch_one<1, 2, 2, 2, false, true>(a, grid, stream);
        else if (a.first)
            e = a.last ? launch_one<2, 2, 1, 2, true, true>(a, grid, stream)
                       : launch_one<2, 2, 1, 2, true, false>(a, grid, stream);
        else
            e = a.last ? launch_one<2, 2, 1, 2, false, true>(a, grid, stream)
                       : launch_one<2, 2, 1, 2, false, false>(a, grid, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace socket_attn
