// Block management on the device: the bookkeeping side of the paged KV cache
// ("从源码剖析 vLLM 的显存管理与连续批处理" §2.1 BlockTable.append_token, §2.2 the
// pool; "vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速" §2.2 Block.ref_count,
// §2.3 sharing by reference count, copy-on-write, reclaim at zero, §3.1 the
// allocation flow; first page §3.2 admission while blocks remain).
//
// State, all caller-owned device memory:
//   ref        int32 [N]   references to each block (0 = free)
//   free_ids   int32 [N]   ring of free block ids: the live entries are the
//                          positions head .. tail-1 (mod N), oldest first
//   free_state int64 [2]   head, tail (positions only grow; tail - head free)
// plus the block tables and context lengths of the attention kernels.
//
// Every operation is one launch of one CTA (up to 1024 threads).  The work is a few
// loads and stores per sequence or block, so a launch costs its latency, not
// bandwidth; one CTA keeps the order of the sequential definition (sequences
// in index order, blocks in logical order, the ring first in first out)
// without any wait on another CTA, so the result is deterministic and equal,
// entry for entry, to the plain sequential bookkeeping.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kBlocksThreads = 1024;

struct BlockState {
    int32_t* ref;
    int32_t* free_ids;
    long long* free_state;  // [0] head, [1] tail
    long long num_blocks;
};

// Exclusive prefix sum over the CTA's threads in thread order; *total gets
// the CTA's sum.  `sh` is shared scratch of 33 values.  Every thread calls it.
template <typename V>
__device__ __forceinline__ V cta_exclusive_scan(V x, V* total, V* sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    V inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const V y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) sh[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const V w = lane < static_cast<int>(blockDim.x >> 5) ? sh[lane] : V(0);
        V winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const V y = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += y;
        }
        sh[lane] = winc - w;
        if (lane == 31) sh[32] = winc;
    }
    __syncthreads();
    const V excl = sh[warp] + inc - x;
    *total = sh[32];
    __syncthreads();  // sh is reused by the next call
    return excl;
}

// ---------------------------------------------------------------- init

__global__ void __launch_bounds__(256) pa_blocks_init_kernel(const __grid_constant__ BlockState st) {
    wait_for_prior_work();
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < st.num_blocks;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        st.free_ids[i] = static_cast<int32_t>(i);
        st.ref[i] = 0;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        st.free_state[0] = 0;
        st.free_state[1] = st.num_blocks;
    }
}

// ---------------------------------------------------------------- append

struct AppendParams {
    int32_t* block_tables;     // [S][MB]
    int32_t* context_lens;     // [S]
    const int32_t* num_new;    // [S] tokens each sequence takes this step
    BlockState st;
    long long* slots;          // [num_slots] packed in sequence order
    long long num_slots;
    long long* pairs;          // [S][2] copy-on-write (old, new) or (-1, -1)
    int num_seqs;
    int max_blocks;
    int block_size;
};

// What sequence s needs this step, read from its row: its length L, token
// count n, the first logical block not yet held, the number of new blocks,
// and X, the partly filled block the first new token falls in (-1 if it
// starts a block).  False when the sequence takes nothing (n == 0) or cannot
// be served because of its own row (error bits set).
__device__ __forceinline__ bool describe_append(const AppendParams& p, int s, int& L, int& n, int& first_new,
                                                int& new_blocks, int& X) {
    L = p.context_lens[s];
    n = p.num_new[s];
    if (n == 0) return false;
    const long long cap = static_cast<long long>(p.max_blocks) * p.block_size;
    if (n < 0 || L < 0 || static_cast<long long>(L) + n > cap) {
        flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
        return false;
    }
    const int B = p.block_size;
    first_new = (L + B - 1) / B;
    new_blocks = static_cast<int>((static_cast<long long>(L) + n + B - 1) / B) - first_new;
    X = -1;
    if (L % B != 0) {
        X = p.block_tables[static_cast<long long>(s) * p.max_blocks + L / B];
        if (X < 0 || X >= p.st.num_blocks) {
            flag_error(1 /* PA_DEVERR_BLOCK_ID */);
            return false;
        }
    }
    return true;
}

// Free-ring entries staged in shared memory at the start (the blocks a step
// takes are the ring's first ones); further entries are read from global memory.
constexpr int kRingWindow = 2048;

// Launched with blockDim.x = a multiple of 32 up to kBlocksThreads (the
// batch rounded up: a small batch syncs few warps).
__global__ void __launch_bounds__(kBlocksThreads) pa_blocks_append_kernel(const __grid_constant__ AppendParams p) {
    wait_for_prior_work();
    __shared__ long long sh[33];
    __shared__ int shx[kBlocksThreads];
    __shared__ int32_t window[kRingWindow];
    __shared__ long long taken_sh;
    const int S = p.num_seqs, B = p.block_size, tid = threadIdx.x, T = blockDim.x;
    const long long N = p.st.num_blocks;
    const long long head = p.st.free_state[0], tail = p.st.free_state[1];
    const long long avail = tail - head;
    long long total;

    // 1. per sequence: its token count (the packed slots must hold all of
    //    them) and whether its first new token falls in a block held by
    //    others (a copy-on-write candidate).  Counts are read before any
    //    change.  The candidates are listed in sequence order in slots[]
    //    (there are at most as many as tokens); pairs[] holds (X, count).
    //    Meanwhile the first entries of the free ring are staged.
    // ring positions are taken modulo N once; later positions wrap by one compare
    const bool ring_ok = head >= 0 && avail >= 0 && avail <= N;
    const long long head_at = ring_ok ? head % N : 0;
    const int win = ring_ok ? static_cast<int>(min(avail, static_cast<long long>(min(kRingWindow, 4 * T)))) : 0;
    if (ring_ok) {
        for (int i = tid; i < win; i += T) {
            const long long at = head_at + i;
            window[i] = p.st.free_ids[at < N ? at : at - N];
        }
    }
    long long tokens = 0, W = 0;
    // A batch of at most T sequences takes one pass per phase with one sequence
    // per thread: step 3 then reuses what step 1 read (kept in registers).
    const bool one_pass = S <= T;
    int rL = 0, rn = 0, rfirst = 0, rnew = 0, rX = -1;
    bool rok = false, rcand = false;
    for (int base = 0; base < S; base += T) {
        const int s = base + tid;
        long long n_tok = 0, cand = 0;
        if (s < S) {
            n_tok = max(p.num_new[s], 0);
            int L = 0, n = 0, first_new = 0, new_blocks = 0, X = -1;
            const bool ok = describe_append(p, s, L, n, first_new, new_blocks, X);
            const int r = ok && X >= 0 ? p.st.ref[X] : 0;
            cand = ok && X >= 0 && r > 1 ? 1 : 0;
            rL = L;
            rn = n;
            rfirst = first_new;
            rnew = new_blocks;
            rX = X;
            rok = ok;
            rcand = cand != 0;
            p.pairs[2 * s] = cand ? X : -1;
            p.pairs[2 * s + 1] = cand ? r : 0;
        }
        const long long at = cta_exclusive_scan<long long>(cand, &total, sh);
        if (cand && W + at < p.num_slots) p.slots[W + at] = s;   // (a step too big for its slots stops below)
        W += total;
        cta_exclusive_scan<long long>(n_tok, &total, sh);
        tokens += total;
    }
    if (tokens > p.num_slots || !ring_ok) {
        if (tid == 0) flag_error(tokens > p.num_slots ? 4 /* PA_DEVERR_SLOT */ : 64 /* PA_DEVERR_REF_COUNT */);
        return;   // uniform: every thread computed the same totals
    }
    if (tid == 0) taken_sh = 0;
    __syncthreads();

    // 2. the k-th writer (in sequence order) into a block of count r copies
    //    it iff k < r - 1: each earlier writer's copy lowered the count by
    //    one, and the last holder writes in place.  Each candidate counts
    //    the earlier ones naming its block (tiles of the list staged in
    //    shared memory); pairs[2s+1] becomes the copy flag.
    for (long long base = 0; base < W; base += T) {
        const long long i = base + tid;
        int s = -1, X = -1, r = 0, k = 0;
        if (i < W) {
            s = static_cast<int>(p.slots[i]);
            X = static_cast<int>(p.pairs[2 * s]);
            r = static_cast<int>(p.pairs[2 * s + 1]);
        }
        for (long long t0 = 0; t0 <= base; t0 += T) {  // tiles of earlier candidates
            __syncthreads();
            const long long j = t0 + tid;
            shx[tid] = j < W ? static_cast<int>(p.pairs[2 * p.slots[j]]) : -1;
            __syncthreads();
            if (i < W) {
                const long long lim = min(static_cast<long long>(T), i - t0);
                for (long long u = 0; u < lim; ++u) k += shx[u] == X;
            }
        }
        __syncthreads();
        if (i < W) p.pairs[2 * s + 1] = k < r - 1 ? 1 : 0;
    }
    __syncthreads();

    // 3. service in sequence order while the free blocks last: with C_s the
    //    running sum of needs (new blocks + a copy), s is served iff
    //    C_s <= free blocks; its blocks are ring positions head + C_s - need_s
    //    onward (the copy first, then new blocks in logical order).
    long long run_need = 0, run_slot = 0;
    const long long cap = static_cast<long long>(p.max_blocks) * B;
    for (int base = 0; base < S; base += T) {
        const int s = base + tid;
        int L = 0, n = 0, first_new = 0, new_blocks = 0, X = -1;
        bool ok = false, cow = false;
        if (s < S && one_pass) {
            L = rL;
            n = rn;
            first_new = rfirst;
            new_blocks = rnew;
            X = rX;
            ok = rok;
            cow = ok && rcand && p.pairs[2 * s + 1] == 1;   // the flag step 2 set
        } else if (s < S) {
            // the row is unchanged since step 1 (only its own thread writes it, below)
            n = p.num_new[s];
            L = p.context_lens[s];
            if (n > 0) {
                ok = L >= 0 && static_cast<long long>(L) + n <= cap;
                if (ok) {
                    first_new = (L + B - 1) / B;
                    new_blocks = static_cast<int>((static_cast<long long>(L) + n + B - 1) / B) - first_new;
                    if (L % B != 0) {
                        X = p.block_tables[static_cast<long long>(s) * p.max_blocks + L / B];
                        ok = X >= 0 && X < N;
                    }
                    cow = ok && X >= 0 && p.pairs[2 * s] >= 0 && p.pairs[2 * s + 1] == 1;
                }
            }
        }
        const long long need = ok ? new_blocks + (cow ? 1 : 0) : 0;
        const long long before = run_need + cta_exclusive_scan<long long>(need, &total, sh);
        run_need += total;
        const long long slot0 = run_slot + cta_exclusive_scan<long long>(s < S ? max(n, 0) : 0, &total, sh);
        run_slot += total;
        if (s >= S) continue;
        const bool served = ok && before + need <= avail;
        if (ok && !served) flag_error(32 /* PA_DEVERR_NO_FREE_BLOCK */);
        int32_t* row = p.block_tables + static_cast<long long>(s) * p.max_blocks;
        if (!served) {
            p.pairs[2 * s] = -1;
            p.pairs[2 * s + 1] = -1;
            for (int i = 0; i < max(n, 0); ++i) p.slots[slot0 + i] = -1;
            continue;
        }
        long long pos = before;   // offset in the ring from head
        auto take = [&]() -> int {
            const long long at = head_at + pos;   // pos < avail <= N
            const int id = pos < win ? window[pos] : p.st.free_ids[at < N ? at : at - N];
            ++pos;
            if (id < 0 || id >= N) {
                flag_error(64 /* PA_DEVERR_REF_COUNT: the ring holds a bad id */);
                return -1;
            }
            p.st.ref[id] = 1;
            return id;
        };
        int c = -1;
        if (cow) {
            c = take();
            atomicSub(p.st.ref + X, 1);
            row[L / B] = c;
            p.pairs[2 * s] = X;
            p.pairs[2 * s + 1] = c;
        } else {
            p.pairs[2 * s] = -1;
            p.pairs[2 * s + 1] = -1;
        }
        if (one_pass) {
            // new blocks taken in logical order as the tokens reach them; each
            // token's slot from the block it lands in (no read-back of the row)
            int cur = L % B != 0 ? (cow ? c : X) : -1;
            int cur_lb = L % B != 0 ? L / B : -1;
            for (int i = 0; i < n; ++i) {
                const int t = L + i;
                if (t / B != cur_lb) {
                    cur_lb = t / B;
                    cur = take();
                    row[cur_lb] = cur;
                }
                p.slots[slot0 + i] = cur < 0 ? -1 : static_cast<long long>(cur) * B + t % B;
            }
        } else {
            for (int j = 0; j < new_blocks; ++j) row[first_new + j] = take();
            for (int i = 0; i < n; ++i) {
                const int t = L + i;
                const int blk = row[t / B];
                p.slots[slot0 + i] = blk < 0 ? -1 : static_cast<long long>(blk) * B + t % B;
            }
        }
        p.context_lens[s] = L + n;
        atomicAdd(reinterpret_cast<unsigned long long*>(&taken_sh), static_cast<unsigned long long>(need));
    }
    __syncthreads();
    if (tid == 0) p.st.free_state[0] = head + taken_sh;
}

// ---------------------------------------------------------------- fork

struct ForkParams {
    int32_t* block_tables;
    int32_t* context_lens;
    int32_t* ref;
    const int32_t* forks;   // [num_forks][3]: parent, child, length
    int num_forks;
    int num_seqs;
    int max_blocks;
    int block_size;
    long long num_blocks;
};

__global__ void __launch_bounds__(kBlocksThreads) pa_blocks_fork_kernel(const __grid_constant__ ForkParams p) {
    wait_for_prior_work();
    __shared__ int parent_sh, child_sh, len_sh, nb_sh;
    const int tid = threadIdx.x;
    for (int k = 0; k < p.num_forks; ++k) {
        if (tid == 0) {
            const int parent = p.forks[3 * k], child = p.forks[3 * k + 1], len = p.forks[3 * k + 2];
            nb_sh = -1;
            if (parent < 0 || parent >= p.num_seqs || child < 0 || child >= p.num_seqs) {
                flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
            } else if (child == parent || p.context_lens[child] != 0) {
                flag_error(64 /* PA_DEVERR_REF_COUNT: the child's own blocks would be lost */);
            } else if (len < 0 || len > p.context_lens[parent] ||
                       static_cast<long long>(len) > static_cast<long long>(p.max_blocks) * p.block_size) {
                flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
            } else {
                parent_sh = parent;
                child_sh = child;
                len_sh = len;
                nb_sh = (len + p.block_size - 1) / p.block_size;
            }
        }
        __syncthreads();
        const int nb = nb_sh;
        if (nb >= 0) {
            const int32_t* from = p.block_tables + static_cast<long long>(parent_sh) * p.max_blocks;
            int32_t* to = p.block_tables + static_cast<long long>(child_sh) * p.max_blocks;
            for (int j = tid; j < nb; j += kBlocksThreads) {
                const int b = from[j];
                to[j] = b;
                if (b >= 0 && b < p.num_blocks) {
                    atomicAdd(p.ref + b, 1);
                } else {
                    flag_error(1 /* PA_DEVERR_BLOCK_ID */);
                }
            }
            __syncthreads();
            if (tid == 0) p.context_lens[child_sh] = len_sh;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- release

struct ReleaseParams {
    int32_t* block_tables;
    int32_t* context_lens;
    BlockState st;
    const int32_t* seqs;    // [num_release] sequences to free, in order
    int num_release;
    int num_seqs;
    int max_blocks;
    int block_size;
};

__global__ void __launch_bounds__(kBlocksThreads) pa_blocks_release_kernel(const __grid_constant__ ReleaseParams p) {
    wait_for_prior_work();
    __shared__ long long sh[33];
    __shared__ int s_sh, nb_sh;
    const int tid = threadIdx.x;
    const long long N = p.st.num_blocks;
    const long long head = p.st.free_state[0], tail = p.st.free_state[1];
    if (head < 0 || tail < head || tail - head > N) {   // not a ring this library wrote
        if (threadIdx.x == 0) flag_error(64 /* PA_DEVERR_REF_COUNT */);
        return;
    }
    const long long tail_at = tail % N;
    long long pushed = 0, total;
    for (int k = 0; k < p.num_release; ++k) {
        if (tid == 0) {
            const int s = p.seqs[k];
            nb_sh = 0;
            if (s < 0 || s >= p.num_seqs) {
                flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
                s_sh = -1;
            } else {
                s_sh = s;
                const int L = p.context_lens[s];
                if (L < 0 || static_cast<long long>(L) > static_cast<long long>(p.max_blocks) * p.block_size) {
                    flag_error(2 /* PA_DEVERR_CONTEXT_LEN */);
                } else {
                    nb_sh = (L + p.block_size - 1) / p.block_size;
                }
            }
        }
        __syncthreads();
        const int s = s_sh, nb = nb_sh;
        if (s >= 0) {
            int32_t* row = p.block_tables + static_cast<long long>(s) * p.max_blocks;
            for (int base = 0; base < nb; base += kBlocksThreads) {
                const int j = base + tid;
                int b = -1;
                long long zero = 0;
                if (j < nb) {
                    b = row[j];
                    if (b < 0 || b >= N) {
                        flag_error(1 /* PA_DEVERR_BLOCK_ID */);
                    } else {
                        const int old = atomicSub(p.st.ref + b, 1);
                        if (old <= 0) {
                            atomicAdd(p.st.ref + b, 1);
                            flag_error(64 /* PA_DEVERR_REF_COUNT */);
                        } else if (old == 1) {
                            zero = 1;  // its count reached zero here: back to the pool
                        }
                    }
                    row[j] = -1;
                }
                const long long at = cta_exclusive_scan<long long>(zero, &total, sh);
                if (zero) {
                    const long long pos = tail + pushed + at;
                    if (pos - head < N) {
                        const long long ring_at = tail_at + pushed + at;   // < 2N
                        p.st.free_ids[ring_at < N ? ring_at : ring_at - N] = b;
                    } else {
                        flag_error(64 /* PA_DEVERR_REF_COUNT: more free blocks than the pool holds */);
                    }
                }
                pushed += total;
            }
            __syncthreads();
            if (tid == 0) p.context_lens[s] = 0;
        }
        __syncthreads();
    }
    if (tid == 0) p.st.free_state[1] = tail + min(pushed, N - (tail - head));
}

}  // namespace pa
