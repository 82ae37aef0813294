// C ABI of the prefix-sliding ring-buffer attention library (see include/ps.h).
//
// Host side: argument validation, the host mirror of every sequence's
// bookkeeping (used only to validate calls and size launches -- the kernels
// read the device copy), and kernel launches.  Nothing is enqueued unless
// every check passed, so a failed call leaves device memory and host state
// untouched.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "ps.h"
#include "internal.h"
#include "page_plan.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int ok() {
  g_err.clear();
  return PS_OK;
}

#define PS_CUDA(expr)                                                                   \
  do {                                                                                  \
    cudaError_t e_ = (expr);                                                            \
    if (e_ != cudaSuccess) return fail(PS_ECUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

struct SeqHost {
  int32_t state;  // 0 empty, 1 active
  int32_t P;
  int64_t next_pos;
  int32_t head;
  int32_t count;
  int32_t owner = -1;   // sequence whose slab holds the prefix rows (itself unless shared)
  int32_t sharers = 0;  // other sequences reading this one's prefix rows
  std::vector<int32_t> pages;  // paged cache: physical page of each ring page (-1: none yet)
};

struct Layout {
  size_t meta, tickets, err, pos, ptab, K, V, total;
};

size_t al(size_t x) { return (x + 255) & ~(size_t)255; }

int esize_of(int dtype) { return dtype == PS_F32 ? 4 : (dtype == PS_BF16 ? 2 : 0); }

// page_rows == 0: unpaged, each sequence's ring inside its own slab
// [Hkv][P_max + W]; otherwise ring pages of page_rows slots come from a pool of
// nphys pages after the prefix slabs [S][Hkv][P_max].
bool make_layout(int W, int P_max, int Hkv, int d, int dtype, int S, int page_rows, int nphys,
                 Layout* L) {
  int es = esize_of(dtype);
  if (W < 1 || W > (1 << 28) || P_max < 0 || P_max > (1 << 28) || Hkv < 1 || Hkv > 1024 ||
      S < 1 || S > (1 << 20) || es == 0)
    return false;
  if (d != 64 && d != 128) return false;
  const bool paged = page_rows > 0;
  if (paged && (page_rows > W || W % page_rows != 0 || nphys < 1 || nphys > (1 << 24)))
    return false;
  const size_t pr = paged ? (size_t)page_rows : (size_t)W;
  const size_t np = paged ? (size_t)nphys : (size_t)S;
  size_t off = 0;
  L->meta = off; off += al((size_t)S * sizeof(ps::DevMeta));
  L->tickets = off; off += al((size_t)S * sizeof(int32_t));
  L->err = off; off += 256;
  L->pos = off; off += al(np * pr * sizeof(int64_t));
  L->ptab = off; off += paged ? al((size_t)S * (W / page_rows) * sizeof(int32_t)) : 0;
  const size_t rows = paged ? (size_t)S * Hkv * P_max + np * Hkv * pr
                            : (size_t)S * Hkv * ((size_t)P_max + W);
  L->K = off; off += al(rows * d * es);
  L->V = off; off += al(rows * d * es);
  L->total = off;
  return true;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace

struct ps_cache {
  int W, P_max, Hkv, d, dtype, S, esize;
  bool paged;
  std::vector<int32_t> free_pages;  // paged: physical ring pages not held by any sequence
  char* base;
  size_t bytes;
  int device;
  int sm_count;
  ps::CacheDev dev;
  ps::DecodeMaps dmaps;  // bf16 caches: tensor maps of K/V for the decode kernel
  int chunk_small_max;   // chunk blocks of at most this many queries: split decode path
  std::vector<SeqHost> seqs;
};

namespace {

int check_device(const ps_cache* c) {
  int cur = -1;
  PS_CUDA(cudaGetDevice(&cur));
  if (cur != c->device)
    return fail(PS_EINVAL, "current device %d is not the cache's device %d", cur, c->device);
  return PS_OK;
}

int check_seq(const ps_cache* c, int seq, bool need_active) {
  if (seq < 0 || seq >= c->S) return fail(PS_EINVAL, "sequence %d out of range [0,%d)", seq, c->S);
  if (need_active && c->seqs[seq].state != 1)
    return fail(PS_ESTATE, "sequence %d has no stored prefix (call ps_prefill_prefix first)", seq);
  return PS_OK;
}

int check_batch(const ps_cache* c, const int* ids, int B) {
  if (B > 0 && !ids) return fail(PS_EINVAL, "seq_ids is NULL");
  std::vector<char> seen(c->S, 0);
  for (int b = 0; b < B; ++b) {
    int r = check_seq(c, ids[b], true);
    if (r) return r;
    if (seen[ids[b]]) return fail(PS_EINVAL, "sequence %d appears twice in the batch", ids[b]);
    seen[ids[b]] = 1;
  }
  return PS_OK;
}

int check_group(const ps_cache* c, int Hq, int* G) {
  if (Hq < 1 || Hq % c->Hkv) return fail(PS_EINVAL, "Hq=%d is not a multiple of Hkv=%d", Hq, c->Hkv);
  *G = Hq / c->Hkv;
  if (*G != 1 && *G != 2 && *G != 4 && *G != 8)
    return fail(PS_EUNSUPPORTED, "Hq/Hkv=%d not in {1,2,4,8}", *G);
  return PS_OK;
}

// Paged cache: page planning for a write to ring slots [slot0, slot0 + n) of
// sequence `seq` (page_plan.h); nothing to do for an unpaged cache.
bool plan_pages(const ps_cache* c, int seq, std::vector<int32_t>& pages, int64_t slot0, int64_t n,
                std::vector<int32_t>& avail, std::vector<int32_t>& idx,
                std::vector<int32_t>& phys) {
  if (!c->paged) return true;
  const ps::PageShape sh{c->W, c->dev.page_rows, c->dev.npg};
  return ps::plan_pages(sh, seq, pages, slot0, n, avail, idx, phys);
}

void advance(SeqHost& s, int W, int64_t n) {
  int64_t cn = (int64_t)s.count + n;
  int64_t adv = cn - W > 0 ? cn - W : 0;
  s.count = (int32_t)(cn < W ? cn : W);
  s.head = (int32_t)(((int64_t)s.head + adv) % W);
  s.next_pos += n;
}

// Records a planned page-table update once its launch is enqueued.  Host
// state follows what is enqueued: if a later launch of the same call fails,
// the mapped pages stay mapped on both sides (the next append that reaches
// them finds them mapped).
void commit_pages(ps_cache* c, const int* seq_ids, int B,
                  const std::vector<std::vector<int32_t>>& pages,
                  const std::vector<int32_t>& avail) {
  if (!c->paged) return;
  c->free_pages = avail;
  for (int b = 0; b < B; ++b) c->seqs[seq_ids[b]].pages = pages[b];
}

ps::DevMeta to_dev(const SeqHost& s) {
  ps::DevMeta m;
  memset(&m, 0, sizeof(m));
  m.next_pos = s.next_pos;
  m.P = s.P;
  m.head = s.head;
  m.count = s.count;
  m.owner = s.owner;
  return m;
}

}  // namespace

// Chunk (prompt == false) or prompt attention of B sequences' blocks, rows
// packed end to end in entry order; then, for chunks with append_after, the
// blocks are appended to the rings.  Everything is validated (and paged ring
// pages planned) before anything is enqueued.
static int attend_blocks(ps_cache* c, const int* seq_ids, const int64_t* t0, const int* n, int B,
                  const void* q, const void* k_blk, const void* v_blk, int Hq, float scale,
                  void* out, int append_after, bool prompt, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (B < 0) return fail(PS_EINVAL, "negative B=%d", B);
  if (B == 0) return ok();
  if (!t0 || !n) return fail(PS_EINVAL, "t0 / n is NULL");
  int r = check_batch(c, seq_ids, B);
  if (r) return r;
  int G = 0;
  if ((r = check_group(c, Hq, &G))) return r;
  int64_t N = 0;
  for (int b = 0; b < B; ++b) {
    const SeqHost& s = c->seqs[seq_ids[b]];
    if (n[b] < 0) return fail(PS_EINVAL, "entry %d: negative n=%d", b, n[b]);
    if (prompt) {
      if (t0[b] < 0 || t0[b] + n[b] > s.P)
        return fail(PS_EPOS, "sequence %d: prompt queries [%lld, %lld) are not inside the prefix (P=%d)",
                    seq_ids[b], (long long)t0[b], (long long)(t0[b] + n[b]), s.P);
    } else {
      if (t0[b] != s.next_pos)
        return fail(PS_EPOS, "sequence %d: t0=%lld does not follow the history (next position %lld)",
                    seq_ids[b], (long long)t0[b], (long long)s.next_pos);
      if (t0[b] < s.P)
        return fail(PS_EPOS, "sequence %d: t0=%lld lies inside the prefix (P=%d)", seq_ids[b],
                    (long long)t0[b], s.P);
    }
    N += n[b];
  }
  if (N > INT32_MAX) return fail(PS_EINVAL, "%lld packed rows exceed 2^31 - 1", (long long)N);
  if (N == 0) return ok();
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(PS_EINVAL, "q/out must be non-NULL 16-byte aligned device pointers");
  if (!prompt && (!k_blk || !v_blk || !aligned16(k_blk) || !aligned16(v_blk)))
    return fail(PS_EINVAL, "k_blk/v_blk must be non-NULL 16-byte aligned device pointers");
  if ((r = check_device(c))) return r;
  // paged: ring pages for the blocks' appended slots, planned before anything runs
  std::vector<int32_t> avail = c->free_pages, idx, phys;
  std::vector<std::vector<int32_t>> pages;
  if (append_after && !prompt) {
    pages.resize(B);
    for (int b = 0; b < B; ++b) {
      const SeqHost& s = c->seqs[seq_ids[b]];
      pages[b] = s.pages;
      const int64_t n_eff = n[b] < c->W ? n[b] : c->W;
      if (n[b] > 0 && !plan_pages(c, seq_ids[b], pages[b],
                                  (int64_t)s.head + s.count + (n[b] - n_eff), n_eff, avail, idx,
                                  phys))
        return fail(PS_ENOMEM, "the ring page pool has no free page left");
    }
  }
  cudaStream_t st = (cudaStream_t)stream;
  const size_t qrow = (size_t)Hq * c->d * c->esize, krow = (size_t)c->Hkv * c->d * c->esize;
  // Small blocks (bf16): groups of a few queries on the tensor-core decode
  // kernel, split over the whole GPU, instead of one 128-row query tile per
  // kv head on the chunk kernel.
  // The whole call takes it when every block is small and their (group, kv
  // head) pairs all fit the GPU at once in clusters of two CTAs; otherwise
  // the chunk kernel's launch takes the small blocks along (its CTAs run
  // them in the same waves).
  std::vector<char> small(B, 0);
  if (!prompt && c->dtype == PS_BF16 && c->chunk_small_max > 0) {
    int nmax = 0;
    int64_t pairs = 0;
    bool all_small = true;
    for (int b = 0; b < B; ++b) {
      if (n[b] == 0) continue;
      if (n[b] > c->chunk_small_max) all_small = false;
      nmax = n[b] > nmax ? n[b] : nmax;
      pairs += (int64_t)((n[b] + 8 / G - 1) / (8 / G)) * c->Hkv;
    }
    if (!all_small || nmax == 0 || pairs > ps::chunk_small_pair_capacity(c->d)) nmax = 0;
    for (int b = 0; b < B; ++b) small[b] = nmax > 0 && n[b] > 0;
    if (nmax > 0) {
      // groups of Q = 8 / G queries: the kernel's 8 columns hold a group's
      // queries x G heads.  Fixed, like the kernel's cluster split, so that an
      // entry's result does not depend on the rest of the batch.
      const int cols = 8;
      const int Q = cols / G;
      std::vector<ps::SmallChunkEntry> es;
      auto flush = [&]() -> cudaError_t {
        if (es.empty()) return cudaSuccess;
        cudaError_t e = ps::launch_chunk_small_batch(c->dev, cols, G, es.data(), (int)es.size(), Hq,
                                                     q, k_blk, v_blk, N, out, scale, c->sm_count,
                                                     c->dmaps, st);
        es.clear();
        return e;
      };
      int64_t tok = 0;
      for (int b = 0; b < B; ++b) {
        if (small[b]) {
          const SeqHost& sh = c->seqs[seq_ids[b]];
          for (int i0 = 0; i0 < n[b]; i0 += Q) {
            ps::SmallChunkEntry e;
            e.seq = seq_ids[b];
            e.P = sh.P;
            e.head = sh.head;
            e.count = sh.count;
            e.owner = sh.owner;
            e.t0 = t0[b];
            e.i0 = i0;
            e.nq = n[b] - i0 < Q ? n[b] - i0 : Q;
            e.qrow = (int32_t)(tok + i0);
            e.brow = (int32_t)tok;
            es.push_back(e);
            if ((int)es.size() == ps::kMaxBatchPerLaunch) PS_CUDA(flush());
          }
        }
        tok += n[b];
      }
      PS_CUDA(flush());
    }
  }
  if (ps::chunk_tc_supported(c->dev, c->dtype, c->d, G)) {
    // entries with queries, in launches of at most kMaxChunkBatch
    std::vector<ps::ChunkEntry> es;
    int64_t tok = 0, tok_first = 0;
    auto flush = [&]() -> cudaError_t {
      if (es.empty()) return cudaSuccess;
      cudaError_t e = ps::launch_chunk_tc(
          c->dev, G, es.data(), (int)es.size(), Hq, (const char*)q + tok_first * qrow,
          prompt ? nullptr : (const char*)k_blk + tok_first * krow,
          prompt ? nullptr : (const char*)v_blk + tok_first * krow, (char*)out + tok_first * qrow,
          scale, prompt ? 1 : 0, c->sm_count, st);
      es.clear();
      return e;
    };
    for (int b = 0; b < B; ++b) {
      if (n[b] > 0 && !small[b]) {
        if (es.empty()) tok_first = tok;
        const SeqHost& sh = c->seqs[seq_ids[b]];
        es.push_back(ps::ChunkEntry{seq_ids[b], n[b], t0[b], sh.next_pos, sh.P, sh.head, sh.count,
                                    sh.owner});
        if ((int)es.size() == ps::kMaxChunkBatch) PS_CUDA(flush());
      } else if (small[b]) {
        PS_CUDA(flush());  // a launch's entries are consecutive in the packed rows
      }
      tok += n[b];
    }
    PS_CUDA(flush());
  } else {
    int64_t tok = 0;
    for (int b = 0; b < B; ++b) {
      if (n[b] > 0 && !small[b])
        PS_CUDA(ps::launch_chunk_cc(
            c->dev, c->dtype, G, seq_ids[b], t0[b], n[b], Hq, (const char*)q + tok * qrow,
            prompt ? nullptr : (const char*)k_blk + tok * krow,
            prompt ? nullptr : (const char*)v_blk + tok * krow, (char*)out + tok * qrow, scale,
            prompt ? 1 : 0, st));
      tok += n[b];
    }
  }
  if (append_after && !prompt) {
    if (!idx.empty())
      PS_CUDA(ps::launch_page_set(c->dev, idx.data(), phys.data(), (int)idx.size(), st));
    commit_pages(c, seq_ids, B, pages, avail);
    int64_t tok = 0;
    for (int b = 0; b < B; ++b) {
      if (n[b] > 0) {
        ps::BatchIds ids;
        memset(&ids, 0, sizeof(ids));
        ids.seq[0] = seq_ids[b];
        PS_CUDA(ps::launch_ring_append(c->dev, c->esize, ids, 1, (const char*)k_blk + tok * krow,
                                       (const char*)v_blk + tok * krow, n[b], st));
        advance(c->seqs[seq_ids[b]], c->W, n[b]);
      }
      tok += n[b];
    }
  }
  return ok();
}

extern "C" {

const char* ps_last_error(void) { return g_err.c_str(); }

const char* ps_version(void) { return "prefix_sliding_window_ring_b200 0.1 (sm_100a)"; }

}  // extern "C"

namespace {

int create_cache(int W, int P_max, int Hkv, int d, int dtype, int max_seqs, int page_rows,
                 int num_pages, void* dev_buf, size_t dev_bytes, void* stream, ps_cache** out) {
  if (!out) return fail(PS_EINVAL, "out is NULL");
  *out = nullptr;
  if (d != 64 && d != 128) return fail(PS_EUNSUPPORTED, "head_dim %d not in {64,128}", d);
  Layout L;
  if (!make_layout(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages, &L))
    return fail(PS_EINVAL,
                "invalid cache shape W=%d P_max=%d Hkv=%d d=%d dtype=%d seqs=%d page_rows=%d "
                "pages=%d",
                W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages);
  if (!dev_buf || ((uintptr_t)dev_buf & 255))
    return fail(PS_EINVAL, "dev_buf must be a non-NULL 256-byte aligned device pointer");
  if (dev_bytes < L.total)
    return fail(PS_ENOMEM, "dev_buf holds %zu bytes, the cache needs %zu", dev_bytes, L.total);
  cudaPointerAttributes attr;
  PS_CUDA(cudaPointerGetAttributes(&attr, dev_buf));
  if (attr.type != cudaMemoryTypeDevice)
    return fail(PS_EINVAL, "dev_buf is not device memory");
  int sm = 0;
  PS_CUDA(cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, attr.device));
  cudaStream_t st = (cudaStream_t)stream;
  PS_CUDA(cudaMemsetAsync(dev_buf, 0, L.total, st));
  const bool paged = page_rows > 0;
  ps_cache* c = new ps_cache();
  c->W = W; c->P_max = P_max; c->Hkv = Hkv; c->d = d; c->dtype = dtype; c->S = max_seqs;
  c->esize = esize_of(dtype);
  c->paged = paged;
  c->base = (char*)dev_buf;
  c->bytes = dev_bytes;
  c->device = attr.device;
  c->sm_count = sm;
  c->dev.meta = (ps::DevMeta*)(c->base + L.meta);
  c->dev.tickets = (int32_t*)(c->base + L.tickets);
  c->dev.err = (int32_t*)(c->base + L.err);
  c->dev.pos = (int64_t*)(c->base + L.pos);
  c->dev.K = c->base + L.K;
  c->dev.V = c->base + L.V;
  c->dev.page_table = paged ? (int32_t*)(c->base + L.ptab) : nullptr;
  c->dev.W = W; c->dev.P_max = P_max; c->dev.Hkv = Hkv; c->dev.d = d; c->dev.S = max_seqs;
  c->dev.page_rows = paged ? page_rows : W;
  c->dev.npg = paged ? W / page_rows : 1;
  c->dev.nphys = paged ? num_pages : max_seqs;
  c->dev.pstride = paged ? P_max : (int64_t)P_max + W;
  c->dev.rstride = paged ? page_rows : (int64_t)P_max + W;
  c->dev.rbase = paged ? (int64_t)max_seqs * Hkv * P_max : P_max;
  if (dtype == PS_BF16 && !ps::make_decode_maps(c->dev, &c->dmaps)) {
    delete c;
    return fail(PS_ECUDA, "tensor-map encoding of the cache's K/V failed");
  }
  c->chunk_small_max = ps::kChunkSmallMaxDefault;
  SeqHost empty{0, 0, 0, 0, 0};
  if (paged) {
    empty.pages.assign(c->dev.npg, -1);
    for (int p = num_pages - 1; p >= 0; --p) c->free_pages.push_back(p);  // page 0 first
  }
  c->seqs.assign(max_seqs, empty);
  *out = c;
  return ok();
}

}  // namespace

extern "C" {

size_t ps_cache_bytes(int W, int P_max, int Hkv, int d, int dtype, int max_seqs) {
  Layout L;
  if (!make_layout(W, P_max, Hkv, d, dtype, max_seqs, 0, 0, &L)) return 0;
  return L.total;
}

size_t ps_cache_bytes_paged(int W, int P_max, int Hkv, int d, int dtype, int max_seqs,
                            int page_rows, int num_pages) {
  Layout L;
  if (page_rows < 1 || !make_layout(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages, &L))
    return 0;
  return L.total;
}

int ps_cache_create(int W, int P_max, int Hkv, int d, int dtype, int max_seqs, void* dev_buf,
                    size_t dev_bytes, void* stream, ps_cache** out) {
  return create_cache(W, P_max, Hkv, d, dtype, max_seqs, 0, 0, dev_buf, dev_bytes, stream, out);
}

int ps_cache_create_paged(int W, int P_max, int Hkv, int d, int dtype, int max_seqs,
                          int page_rows, int num_pages, void* dev_buf, size_t dev_bytes,
                          void* stream, ps_cache** out) {
  if (page_rows < 1) {
    if (out) *out = nullptr;
    return fail(PS_EINVAL, "page_rows=%d must be at least 1", page_rows);
  }
  return create_cache(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages, dev_buf,
                      dev_bytes, stream, out);
}

int ps_ring_pages_free(const ps_cache* c) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (!c->paged) return fail(PS_EINVAL, "the cache is not paged");
  return (int)c->free_pages.size();
}

void ps_cache_destroy(ps_cache* c) { delete c; }

int ps_seq_info_get(const ps_cache* c, int seq, ps_seq_info* out) {
  if (!c || !out) return fail(PS_EINVAL, "NULL argument");
  int r = check_seq(c, seq, false);
  if (r) return r;
  const SeqHost& s = c->seqs[seq];
  out->state = s.state; out->P = s.P; out->next_pos = s.next_pos;
  out->head = s.head; out->count = s.count;
  return ok();
}

int ps_seq_reset(ps_cache* c, int seq, int ring_head_offset, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, false);
  if (r) return r;
  if (ring_head_offset < 0 || ring_head_offset >= c->W)
    return fail(PS_EINVAL, "ring_head_offset %d not in [0,%d)", ring_head_offset, c->W);
  const SeqHost cur = c->seqs[seq];
  if (cur.sharers > 0)
    return fail(PS_ESTATE, "sequence %d's prefix is read by %d other sequences (reset them first)",
                seq, cur.sharers);
  if ((r = check_device(c))) return r;
  SeqHost s{0, 0, 0, ring_head_offset, 0};
  s.owner = seq;
  PS_CUDA(ps::launch_meta_set(c->dev, seq, to_dev(s), (cudaStream_t)stream));
  if (cur.state == 1 && cur.owner >= 0 && cur.owner != seq) c->seqs[cur.owner].sharers--;
  if (c->paged) {  // its ring pages go back to the pool
    for (int32_t p : cur.pages)
      if (p >= 0) c->free_pages.push_back(p);
    s.pages.assign(c->dev.npg, -1);
  }
  c->seqs[seq] = s;
  return ok();
}

int ps_prefill_prefix(ps_cache* c, int seq, const void* k, const void* v, int P_s, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, false);
  if (r) return r;
  if (c->seqs[seq].state != 0)
    return fail(PS_ESTATE, "sequence %d already has a prefix (reset it first)", seq);
  if (P_s < 0 || P_s > c->P_max) return fail(PS_EINVAL, "P_s=%d not in [0,%d]", P_s, c->P_max);
  if (P_s > 0 && (!k || !v || !aligned16(k) || !aligned16(v)))
    return fail(PS_EINVAL, "k/v must be non-NULL 16-byte aligned device pointers");
  if ((r = check_device(c))) return r;
  cudaStream_t st = (cudaStream_t)stream;
  PS_CUDA(ps::launch_prefix_store(c->dev, c->esize, seq, k, v, P_s, st));
  SeqHost s = c->seqs[seq];
  s.state = 1; s.P = P_s; s.next_pos = P_s; s.count = 0; s.owner = seq;
  PS_CUDA(ps::launch_meta_set(c->dev, seq, to_dev(s), st));
  c->seqs[seq] = s;
  return ok();
}

int ps_share_prefix(ps_cache* c, int seq, int src, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, false);
  if (r) return r;
  if ((r = check_seq(c, src, true))) return r;
  if (seq == src) return fail(PS_EINVAL, "sequence %d cannot share its own prefix", seq);
  if (c->seqs[seq].state != 0)
    return fail(PS_ESTATE, "sequence %d already has a prefix (reset it first)", seq);
  if ((r = check_device(c))) return r;
  const int owner = c->seqs[src].owner;
  SeqHost s = c->seqs[seq];
  s.state = 1; s.P = c->seqs[src].P; s.next_pos = s.P; s.count = 0; s.owner = owner;
  s.sharers = 0;
  PS_CUDA(ps::launch_meta_set(c->dev, seq, to_dev(s), (cudaStream_t)stream));
  c->seqs[seq] = s;
  c->seqs[owner].sharers++;
  return ok();
}

int ps_append_kv(ps_cache* c, const int* seq_ids, int B, const void* k, const void* v, int n,
                 void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (B < 0 || n < 0) return fail(PS_EINVAL, "negative B=%d or n=%d", B, n);
  if (B == 0 || n == 0) return ok();
  int r = check_batch(c, seq_ids, B);
  if (r) return r;
  if (!k || !v || !aligned16(k) || !aligned16(v))
    return fail(PS_EINVAL, "k/v must be non-NULL 16-byte aligned device pointers");
  if ((r = check_device(c))) return r;
  // paged: ring pages for the slots the appends write (the last min(n, W) tokens)
  std::vector<int32_t> avail = c->free_pages, idx, phys;
  std::vector<std::vector<int32_t>> pages(B);
  for (int b = 0; b < B; ++b) {
    const SeqHost& s = c->seqs[seq_ids[b]];
    pages[b] = s.pages;
    const int64_t n_eff = n < c->W ? n : c->W;
    if (!plan_pages(c, seq_ids[b], pages[b], (int64_t)s.head + s.count + (n - n_eff), n_eff,
                    avail, idx, phys))
      return fail(PS_ENOMEM, "the ring page pool has no free page left");
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (!idx.empty())
    PS_CUDA(ps::launch_page_set(c->dev, idx.data(), phys.data(), (int)idx.size(), st));
  commit_pages(c, seq_ids, B, pages, avail);
  size_t per_entry = (size_t)n * c->Hkv * c->d * c->esize;
  for (int b0 = 0; b0 < B; b0 += ps::kMaxBatchPerLaunch) {
    int nb = B - b0 < ps::kMaxBatchPerLaunch ? B - b0 : ps::kMaxBatchPerLaunch;
    ps::BatchIds ids;
    memset(&ids, 0, sizeof(ids));
    for (int i = 0; i < nb; ++i) ids.seq[i] = seq_ids[b0 + i];
    PS_CUDA(ps::launch_ring_append(c->dev, c->esize, ids, nb, (const char*)k + b0 * per_entry,
                                   (const char*)v + b0 * per_entry, n, st));
    for (int i = 0; i < nb; ++i) advance(c->seqs[seq_ids[b0 + i]], c->W, n);
  }
  return ok();
}

size_t ps_decode_workspace_bytes(const ps_cache* c, int B, int Hq) {
  if (!c || B < 0 || Hq < 1 || Hq % c->Hkv) return 0;
  return ps::decode_workspace_bytes(B, Hq, c->Hkv, c->d, c->sm_count);
}

int ps_attend_decode(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t, int B,
                     int Hq, float scale, void* out, void* workspace, size_t workspace_bytes,
                     void* stream) {
  int G = 0;
  int r = ps::check_decode_call(c, q, seq_ids, t, B, Hq, out, &G);
  if (r) return r;
  if (B == 0) return ok();
  if (!workspace || ((uintptr_t)workspace & 255))
    return fail(PS_EINVAL, "workspace must be a non-NULL 256-byte aligned device pointer");
  size_t need = 0;
  ps::DecodeWs ws = ps::decode_ws_layout(workspace, B, c->Hkv, G, c->d, c->sm_count, &need);
  if (need > workspace_bytes)
    return fail(PS_ENOMEM, "workspace holds %zu bytes, this call needs %zu", workspace_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  size_t per_entry = (size_t)Hq * c->d * c->esize;
  for (int b0 = 0; b0 < B; b0 += ps::kMaxBatchPerLaunch) {
    int nb = B - b0 < ps::kMaxBatchPerLaunch ? B - b0 : ps::kMaxBatchPerLaunch;
    ps::BatchIds ids;
    memset(&ids, 0, sizeof(ids));
    for (int i = 0; i < nb; ++i) {
      const SeqHost& s = c->seqs[seq_ids[b0 + i]];
      ids.seq[i] = seq_ids[b0 + i];
      ids.P[i] = s.P;
      ids.head[i] = s.head;
      ids.count[i] = s.count;
      ids.owner[i] = s.owner;
      ids.t[i] = t[b0 + i];
    }
    PS_CUDA(ps::launch_decode(c->dev, c->dtype, G, ids, nb, Hq, (const char*)q + b0 * per_entry,
                              nullptr, nullptr, (char*)out + b0 * per_entry, scale, ws,
                              c->sm_count, c->dtype == PS_BF16 ? &c->dmaps : nullptr, st));
  }
  return ok();
}

int ps_decode_step(ps_cache* c, const void* q, const void* k_new, const void* v_new,
                   const int* seq_ids, const int64_t* t, int B, int Hq, float scale, void* out,
                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (B < 0) return fail(PS_EINVAL, "negative B=%d", B);
  int G = 0;
  int r = check_group(c, Hq, &G);
  if (r) return r;
  if (B == 0) return ok();
  if ((r = check_batch(c, seq_ids, B))) return r;
  if (!t) return fail(PS_EINVAL, "t is NULL");
  for (int b = 0; b < B; ++b) {
    const SeqHost& s = c->seqs[seq_ids[b]];
    if (t[b] != s.next_pos)
      return fail(PS_EPOS, "sequence %d: t=%lld is not the next position %lld", seq_ids[b],
                  (long long)t[b], (long long)s.next_pos);
    if (t[b] < s.P)
      return fail(PS_EPOS, "sequence %d: t=%lld lies inside the prefix (P=%d)", seq_ids[b],
                  (long long)t[b], s.P);
  }
  if (!q || !out || !k_new || !v_new || !aligned16(q) || !aligned16(out) || !aligned16(k_new) ||
      !aligned16(v_new))
    return fail(PS_EINVAL, "q/k_new/v_new/out must be non-NULL 16-byte aligned device pointers");
  if (!workspace || ((uintptr_t)workspace & 255))
    return fail(PS_EINVAL, "workspace must be a non-NULL 256-byte aligned device pointer");
  size_t need = 0;
  ps::DecodeWs ws = ps::decode_ws_layout(workspace, B, c->Hkv, G, c->d, c->sm_count, &need);
  if (need > workspace_bytes)
    return fail(PS_ENOMEM, "workspace holds %zu bytes, this call needs %zu", workspace_bytes, need);
  if ((r = check_device(c))) return r;
  // paged: a ring page for each appended token's slot
  std::vector<int32_t> avail = c->free_pages, idx, phys;
  std::vector<std::vector<int32_t>> pages(B);
  for (int b = 0; b < B; ++b) {
    const SeqHost& s = c->seqs[seq_ids[b]];
    pages[b] = s.pages;
    if (!plan_pages(c, seq_ids[b], pages[b], (int64_t)s.head + s.count, 1, avail, idx, phys))
      return fail(PS_ENOMEM, "the ring page pool has no free page left");
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (!idx.empty())
    PS_CUDA(ps::launch_page_set(c->dev, idx.data(), phys.data(), (int)idx.size(), st));
  commit_pages(c, seq_ids, B, pages, avail);
  const size_t per_entry = (size_t)Hq * c->d * c->esize;
  const size_t per_row = (size_t)c->Hkv * c->d * c->esize;
  for (int b0 = 0; b0 < B; b0 += ps::kMaxBatchPerLaunch) {
    int nb = B - b0 < ps::kMaxBatchPerLaunch ? B - b0 : ps::kMaxBatchPerLaunch;
    ps::BatchIds ids;
    memset(&ids, 0, sizeof(ids));
    for (int i = 0; i < nb; ++i) {
      SeqHost s = c->seqs[seq_ids[b0 + i]];
      advance(s, c->W, 1);  // the state the attention sees: the token appended
      ids.seq[i] = seq_ids[b0 + i];
      ids.P[i] = s.P;
      ids.head[i] = s.head;
      ids.count[i] = s.count;
      ids.owner[i] = s.owner;
      ids.t[i] = t[b0 + i];
    }
    PS_CUDA(ps::launch_decode(c->dev, c->dtype, G, ids, nb, Hq, (const char*)q + b0 * per_entry,
                              (const char*)k_new + b0 * per_row, (const char*)v_new + b0 * per_row,
                              (char*)out + b0 * per_entry, scale, ws, c->sm_count,
                              c->dtype == PS_BF16 ? &c->dmaps : nullptr, st));
    for (int i = 0; i < nb; ++i) advance(c->seqs[seq_ids[b0 + i]], c->W, 1);
  }
  return ok();
}

int ps_set_chunk_small_max(ps_cache* c, int n_max) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (n_max < 0) return fail(PS_EINVAL, "negative n_max=%d", n_max);
  c->chunk_small_max = n_max;
  return ok();
}

int ps_attend_chunk(ps_cache* c, int seq, const void* q, const void* k_blk, const void* v_blk,
                    int64_t t0, int n, int Hq, float scale, void* out, int append_after,
                    void* stream) {
  return attend_blocks(c, &seq, &t0, &n, 1, q, k_blk, v_blk, Hq, scale, out, append_after, false,
                       stream);
}

int ps_attend_chunk_batch(ps_cache* c, const int* seq_ids, const int64_t* t0, const int* n, int B,
                          const void* q, const void* k_blk, const void* v_blk, int Hq,
                          float scale, void* out, int append_after, void* stream) {
  return attend_blocks(c, seq_ids, t0, n, B, q, k_blk, v_blk, Hq, scale, out, append_after, false,
                       stream);
}

int ps_attend_prompt(ps_cache* c, int seq, const void* q, int64_t t0, int n, int Hq, float scale,
                     void* out, void* stream) {
  return attend_blocks(c, &seq, &t0, &n, 1, q, nullptr, nullptr, Hq, scale, out, 0, true, stream);
}

int ps_attend_prompt_batch(ps_cache* c, const int* seq_ids, const int64_t* t0, const int* n, int B,
                           const void* q, int Hq, float scale, void* out, void* stream) {
  return attend_blocks(c, seq_ids, t0, n, B, q, nullptr, nullptr, Hq, scale, out, 0, true,
                       stream);
}

int ps_export_window(ps_cache* c, int seq, void* k, void* v, int64_t* pos, int32_t* count_out,
                     void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, true);
  if (r) return r;
  if (!k || !v || !pos || !count_out || !aligned16(k) || !aligned16(v) || ((uintptr_t)pos & 7) ||
      ((uintptr_t)count_out & 3))
    return fail(PS_EINVAL, "k/v/pos/count_out must be non-NULL aligned device pointers");
  if ((r = check_device(c))) return r;
  PS_CUDA(ps::launch_ring_export(c->dev, c->esize, seq, k, v, pos, count_out,
                                 (cudaStream_t)stream));
  return ok();
}

int ps_import_window(ps_cache* c, int seq, int64_t next_pos, const void* k, const void* v, int n,
                     int ring_head_offset, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, true);
  if (r) return r;
  SeqHost s = c->seqs[seq];
  if (next_pos < s.P)
    return fail(PS_EPOS, "next_pos=%lld lies inside the prefix (P=%d)", (long long)next_pos, s.P);
  int64_t want = next_pos - s.P < c->W ? next_pos - s.P : c->W;
  if (n != want)
    return fail(PS_EPOS, "n=%d rows given, the window of next_pos=%lld holds %lld", n,
                (long long)next_pos, (long long)want);
  if (ring_head_offset < 0 || ring_head_offset >= c->W)
    return fail(PS_EINVAL, "ring_head_offset %d not in [0,%d)", ring_head_offset, c->W);
  if (n > 0 && (!k || !v || !aligned16(k) || !aligned16(v)))
    return fail(PS_EINVAL, "k/v must be non-NULL 16-byte aligned device pointers");
  if ((r = check_device(c))) return r;
  std::vector<int32_t> avail = c->free_pages, idx, phys;
  if (!plan_pages(c, seq, s.pages, ring_head_offset, n, avail, idx, phys))
    return fail(PS_ENOMEM, "the ring page pool has no free page left");
  if (!idx.empty())
    PS_CUDA(ps::launch_page_set(c->dev, idx.data(), phys.data(), (int)idx.size(),
                                (cudaStream_t)stream));
  c->free_pages = avail;  // the page-table update is enqueued
  c->seqs[seq].pages = s.pages;
  s.next_pos = next_pos;
  s.head = ring_head_offset;
  s.count = n;
  PS_CUDA(ps::launch_ring_import(c->dev, c->esize, seq, to_dev(s), k, v, n,
                                 (cudaStream_t)stream));
  c->seqs[seq] = s;
  return ok();
}

int ps_debug_visible(ps_cache* c, int seq, int64_t t, int64_t* pos_out, int32_t* n_out,
                     void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  int r = check_seq(c, seq, true);
  if (r) return r;
  const SeqHost& s = c->seqs[seq];
  if (t < s.P) return fail(PS_EPOS, "t=%lld lies inside the prefix (P=%d)", (long long)t, s.P);
  int64_t lo = t - c->W + 1 > s.P ? t - c->W + 1 : s.P;
  int64_t base = s.next_pos - s.count;
  if (lo < base && lo <= s.next_pos - 1)
    return fail(PS_EPOS, "window of t=%lld starts at %lld, the ring holds from %lld",
                (long long)t, (long long)lo, (long long)base);
  if (!pos_out || !n_out || ((uintptr_t)pos_out & 7) || ((uintptr_t)n_out & 3))
    return fail(PS_EINVAL, "pos_out/n_out must be non-NULL aligned device pointers");
  if ((r = check_device(c))) return r;
  PS_CUDA(ps::launch_debug_visible(c->dev, seq, t, pos_out, n_out, (cudaStream_t)stream));
  return ok();
}

int ps_debug_wait_timeout(ps_cache* c, long long limit_cycles, void* stream) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (limit_cycles < 1 || limit_cycles > (1ll << 31))
    return fail(PS_EINVAL, "limit_cycles=%lld outside [1, 2^31]", limit_cycles);
  int r = check_device(c);
  if (r) return r;
  PS_CUDA(ps::launch_debug_wait_timeout(c->dev, limit_cycles, (cudaStream_t)stream));
  return ok();
}

int ps_device_error(ps_cache* c, int32_t* code, void* stream) {
  if (!c || !code) return fail(PS_EINVAL, "NULL argument");
  int r = check_device(c);
  if (r) return r;
  cudaStream_t st = (cudaStream_t)stream;
  PS_CUDA(cudaStreamSynchronize(st));
  int32_t v = 0;
  PS_CUDA(cudaMemcpy(&v, c->dev.err, sizeof(v), cudaMemcpyDeviceToHost));
  PS_CUDA(cudaMemset(c->dev.err, 0, sizeof(int32_t)));
  *code = v;
  return ok();
}

}  // extern "C"

namespace ps {

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int check_decode_call(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t, int B,
                      int Hq, const void* out, int* G) {
  if (!c) return fail(PS_EINVAL, "cache is NULL");
  if (B < 0) return fail(PS_EINVAL, "negative B=%d", B);
  int r = check_group(c, Hq, G);
  if (r) return r;
  if (B == 0) return PS_OK;
  if ((r = check_batch(c, seq_ids, B))) return r;
  if (!t) return fail(PS_EINVAL, "t is NULL");
  for (int b = 0; b < B; ++b) {
    const SeqHost& s = c->seqs[seq_ids[b]];
    if (t[b] != s.next_pos - 1)
      return fail(PS_EPOS, "sequence %d: t=%lld is not the last appended position %lld",
                  seq_ids[b], (long long)t[b], (long long)(s.next_pos - 1));
    if (t[b] < s.P)
      return fail(PS_EPOS, "sequence %d: t=%lld lies inside the prefix (P=%d); append first",
                  seq_ids[b], (long long)t[b], s.P);
  }
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(PS_EINVAL, "q/out must be non-NULL 16-byte aligned device pointers");
  return check_device(c);
}

int cache_hkv(const ps_cache* c) { return c->Hkv; }
int cache_head_dim(const ps_cache* c) { return c->d; }
int cache_sm_count(const ps_cache* c) { return c->sm_count; }

}  // namespace ps
