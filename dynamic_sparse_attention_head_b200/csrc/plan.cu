// Host side of libmsa: problem validation, row classes, estimation row sets, workspace
// layout, tensor maps, and the C entry points declared in include/msa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <tuple>
#include <new>
#include <vector>

#include "kernels.h"
#include "msa_internal.h"

using namespace msa;

#include <atomic>

namespace msa {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace msa

struct msa_plan {
  int64_t L = 0;
  int32_t Hq = 0, Hkv = 0;
  float scale = 0.f;
  std::vector<msa_segment> segs;
  std::vector<msa_head_cfg> heads;
  std::vector<uint8_t> mod;
  std::vector<int32_t> rank;
  int64_t n_mod[2] = {0, 0};
  std::vector<ClassStatic> classes;
  std::vector<HeadStatic> hs;
  std::vector<RowSet> rowsets;
  std::vector<LqTile> lqtiles;
  std::vector<TopkJob> jobs;
  std::vector<WorkItem> items;
  std::vector<UnitBand> bands;
  std::vector<int32_t> segtab;
  Layout lay{};
  DevPlan dp{};
  int32_t n_kchunks = 1, chunk_keys = 0, n_units = 0, band_cap = 0;
  int64_t blob_bytes = 0;
  std::vector<uint8_t> blob;
  int64_t total_tiles = 0;
  std::vector<int32_t> class_kind;
  const void* ready_ws = nullptr;  // workspace holding this plan's indices
};

namespace {

inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct Bump {
  int64_t off = 0;
  int64_t take(int64_t bytes, int64_t align = 256) {
    off = round_up(off, align);
    int64_t r = off;
    off += std::max<int64_t>(bytes, 0);
    return r;
  }
};

int32_t budget_scale(int32_t k, int64_t n, int64_t L) {
  if (n <= 0) return 0;
  int64_t r = (2 * (int64_t)k * n + L) / (2 * L);
  return (int32_t)std::max<int64_t>(1, r);
}

int32_t phases_for(const msa_head_cfg& h, int32_t s) {
  int32_t n = h.n_phases > 0 ? h.n_phases : std::max(1, (int32_t)std::floor(h.grid_budget * s / 2.0));
  return std::min(n, s);
}

msa_status validate(const msa_problem* p) {
  if (!p || !p->segments || !p->heads) return MSA_ERR_INVALID_ARG;
  if (p->d != D) return MSA_ERR_SHAPE;
  if (p->L < 64 || p->L % 64 != 0) return MSA_ERR_SHAPE;
  if (p->L >= (int64_t(1) << 27)) return MSA_ERR_UNSUPPORTED;  // tile rows use 28 bits
  if (p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv != 0) return MSA_ERR_SHAPE;
  if (!(p->scale > 0.f) || !std::isfinite(p->scale)) return MSA_ERR_INVALID_ARG;
  if (p->n_segments <= 0) return MSA_ERR_SHAPE;
  int64_t pos = 0;
  for (int i = 0; i < p->n_segments; ++i) {
    const msa_segment& s = p->segments[i];
    if (s.start != pos || s.len <= 0) return MSA_ERR_SHAPE;
    if (s.modality != MSA_TEXT && s.modality != MSA_VIDEO) return MSA_ERR_INVALID_ARG;
    pos += s.len;
  }
  if (pos != p->L) return MSA_ERR_SHAPE;
  for (int h = 0; h < p->Hq; ++h) {
    const msa_head_cfg& c = p->heads[h];
    if (c.kind < MSA_DENSE || c.kind > MSA_BOUND2D) return MSA_ERR_INVALID_ARG;
    if (c.sink < 0 || c.local < 0 || c.k_v < 0 || c.k_s < 0 || c.topk_blocks < 0) return MSA_ERR_INVALID_ARG;
    if (c.kind == MSA_VSLASH || c.kind == MSA_QBOUND || c.kind == MSA_BOUND2D)
      if (c.k_v < 1 || c.k_s < 1) return MSA_ERR_INVALID_ARG;
    if (c.kind == MSA_BLOCK && c.topk_blocks == 0 && !(c.block_budget > 0.0)) return MSA_ERR_INVALID_ARG;
    if ((c.flags & ~MSA_HEAD_PER_SEGMENT) || ((c.flags & MSA_HEAD_PER_SEGMENT) && c.kind != MSA_QBOUND))
      return MSA_ERR_INVALID_ARG;
    if (c.kind == MSA_GRID) {
      if (c.n_strides < 1 || c.n_strides > MSA_MAX_STRIDES) return MSA_ERR_INVALID_ARG;
      for (int i = 0; i < c.n_strides; ++i)
        if (c.strides[i] < 1) return MSA_ERR_INVALID_ARG;
        else if (c.strides[i] > 4096) return MSA_ERR_UNSUPPORTED;
      if (c.n_phases < 0 || (c.n_phases == 0 && !(c.grid_budget > 0.0))) return MSA_ERR_INVALID_ARG;
    }
  }
  return MSA_OK;
}

// last n positions of modality a (or of the whole sequence when a < 0)
std::vector<int32_t> last_rows(const msa_plan& P, int a, int n = LASTQ) {
  std::vector<int32_t> r;
  for (int64_t t = P.L - 1; t >= 0 && (int)r.size() < n; --t)
    if (a < 0 || P.mod[t] == a) r.push_back((int32_t)t);
  std::reverse(r.begin(), r.end());
  return r;
}

}  // namespace

extern "C" {

uint64_t msa_kernel_launches(void) { return msa::g_launches.load(std::memory_order_relaxed); }

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_SHAPE: return "bad shape (d must be 128, L a multiple of 64, Hq a multiple of Hkv, segments tiling [0, L))";
    case MSA_ERR_ALIGN: return "misaligned pointer or stride (16-byte pointers, strides multiple of 8 elements, 256-byte workspace)";
    case MSA_ERR_WORKSPACE: return "workspace smaller than msa_workspace_bytes()";
    case MSA_ERR_UNSUPPORTED: return "outside this build's limits (L < 2^27, grid stride <= 4096, estimation rows spanning <= 4096 positions)";
    case MSA_ERR_CUDA: return "CUDA call failed";
    case MSA_ERR_TIMEOUT: return "device: a bounded wait expired";
    case MSA_ERR_DEVICE_BOUNDS: return "device: an index fell outside its buffer";
    case MSA_ERR_STATE: return "calls out of order: run msa_estimate or msa_set_indices on this workspace first";
  }
  return "unknown status";
}

msa_status msa_plan_create(const msa_problem* prob, msa_plan** out) {
  if (!out) return MSA_ERR_INVALID_ARG;
  *out = nullptr;
  msa_status st = validate(prob);
  if (st != MSA_OK) return st;
  msa_plan* P = new (std::nothrow) msa_plan();
  if (!P) return MSA_ERR_INVALID_ARG;
  P->L = prob->L;
  P->Hq = prob->Hq;
  P->Hkv = prob->Hkv;
  P->scale = prob->scale;
  P->segs.assign(prob->segments, prob->segments + prob->n_segments);
  P->heads.assign(prob->heads, prob->heads + prob->Hq);
  const int64_t L = P->L;
  const int32_t Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv;
  const int64_t nb = L / BLK;
  const int64_t nwords = (L + 31) / 32;
  // rows of a head's permuted Q / O slice: classes start at multiples of 128 rows; a head with
  // one class per segment needs the segments' lengths rounded up
  int64_t lp = round_up(L, TILE) + 2 * TILE;
  for (int32_t h = 0; h < prob->Hq; ++h)
    if (prob->heads[h].flags & MSA_HEAD_PER_SEGMENT) {
      int64_t r = 2 * TILE;
      for (int i = 0; i < prob->n_segments; ++i) r += round_up(prob->segments[i].len, TILE);
      lp = std::max(lp, r);
    }
  const int32_t LP = (int32_t)lp;
  P->mod.assign(L, 0);
  P->rank.assign(L, 0);
  for (const auto& s : P->segs)
    for (int64_t t = s.start; t < s.start + s.len; ++t) P->mod[t] = (uint8_t)s.modality;
  for (int64_t t = 0; t < L; ++t) P->rank[t] = (int32_t)(P->n_mod[P->mod[t]]++);
  for (const auto& s : P->segs) {
    P->segtab.push_back((int32_t)s.start);
    P->segtab.push_back((int32_t)s.len);
    P->segtab.push_back(s.modality);
  }
  const int64_t region0[2] = {0, P->n_mod[0]};  // modality-grouped order: text, then video

  Bump B;
  Layout& lay = P->lay;
  // sizes of the blob tables first (counts need the class construction below)
  std::vector<ClassStatic>& C = P->classes;
  std::vector<HeadStatic>& HS = P->hs;
  HS.assign(Hq, HeadStatic{});
  bool has2d = false, has_block = false;
  int n_qslices = 0, n_xslices = 0;
  int32_t x_rows_max = 0;

  // ---- classes per head
  for (int32_t h = 0; h < Hq; ++h) {
    const msa_head_cfg& cfg = P->heads[h];
    HeadStatic& H = HS[h];
    H.kind = cfg.kind;
    H.kvh = h / G;
    H.class0 = (int32_t)C.size();
    H.q_slice = -1;
    H.x_slice = -1;
    auto base = [&](int32_t flags) {
      ClassStatic c{};
      c.head = h;
      c.kvh = H.kvh;
      c.kind = cfg.kind;
      c.flags = flags;
      c.k_src = SRC_K;
      c.kc_lo = 0;
      c.kc_hi = (int32_t)L;
      c.krow_lo = 0;
      c.max_rows = (int32_t)L;
      c.rows_static = (int32_t)L;
      c.qrow0_static = 0;
      c.seg = -1;
      return c;
    };
    switch (cfg.kind) {
      case MSA_DENSE: C.push_back(base(CF_DENSE)); break;
      case MSA_ASHAPE: {
        int32_t f = 0;
        if (cfg.sink > 0) f |= CF_SINK;
        if (cfg.local > 0) f |= CF_BAND;
        ClassStatic c = base(f);
        c.sink = cfg.sink;
        c.band = cfg.local;
        C.push_back(c);
        break;
      }
      case MSA_VSLASH: {
        ClassStatic c = base(CF_X | CF_SLASH | CF_EXCL);
        c.x_cap = (int32_t)round_up(std::min<int64_t>(cfg.k_v, L), TILE);
        C.push_back(c);
        break;
      }
      case MSA_BLOCK: {
        ClassStatic c = base(CF_BLOCK);
        c.blk_wpr = (int32_t)((nb + 31) / 32);
        C.push_back(c);
        has_block = true;
        break;
      }
      case MSA_GRID: {
        // rows on grid lines + text rows: dense; other video rows: gathered grid keys + local band
        ClassStatic c0 = base(CF_PERMUTED | CF_DENSE | CF_DYNROWS);
        c0.modality = 0;
        c0.rows_static = -1;
        ClassStatic c1 = base(CF_PERMUTED | CF_DYNROWS | CF_X | CF_BAND | CF_EXCL);
        c1.modality = 1;
        c1.rows_static = -1;
        c1.band = cfg.local > 0 ? cfg.local : GRID_BAND;
        int64_t gmax = 0;
        for (int i = 0; i < cfg.n_strides; ++i) {
          int32_t s = cfg.strides[i], np = phases_for(cfg, s);
          int64_t g = 0;
          for (const auto& sg : P->segs)
            if (sg.modality == MSA_VIDEO) g += std::min<int64_t>(sg.len, (int64_t)np * ((sg.len + s - 1) / s));
          gmax = std::max(gmax, g);
        }
        c1.x_cap = (int32_t)round_up(std::max<int64_t>(gmax, 1), TILE);
        C.push_back(c0);
        C.push_back(c1);
        // candidates in ascending order: on equal best-phase means the smaller stride wins
        std::vector<int32_t> cand(cfg.strides, cfg.strides + cfg.n_strides);
        std::sort(cand.begin(), cand.end());
        cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
        H.grid_n_cand = (int32_t)cand.size();
        for (int i = 0; i < H.grid_n_cand; ++i) {
          H.grid_cand[i] = cand[i];
          H.grid_np[i] = phases_for(cfg, cand[i]);
        }
        H.grid_band = c1.band;
        break;
      }
      case MSA_QBOUND:
        if (cfg.flags & MSA_HEAD_PER_SEGMENT) {
          // one class per segment: its queries (a contiguous run of its modality's positions)
          // with their own vertical and slash lines
          int32_t q0 = 0;
          for (int k = 0; k < (int)P->segs.size(); ++k) {
            const msa_segment& sg = P->segs[k];
            ClassStatic c = base(CF_PERMUTED | CF_X | CF_SLASH | CF_EXCL | CF_SEGIDX);
            c.modality = sg.modality;
            c.seg = k;
            c.max_rows = c.rows_static = (int32_t)sg.len;
            c.qrow0_static = q0;
            q0 += (int32_t)round_up(sg.len, TILE);
            c.x_cap = (int32_t)round_up(std::min<int64_t>(cfg.k_v, L), TILE);
            c.segv_cap = (int32_t)std::min<int64_t>(cfg.k_v, L);
            c.segs_cap = (int32_t)std::min<int64_t>(cfg.k_s, L);
            C.push_back(c);
          }
          break;
        }
        [[fallthrough]];
      case MSA_BOUND2D: {
        const bool two = cfg.kind == MSA_BOUND2D;
        for (int a = 0; a < 2; ++a) {
          if (P->n_mod[a] == 0) continue;
          ClassStatic c = base(CF_PERMUTED | CF_X | CF_SLASH | CF_EXCL | (two ? CF_RANK : 0));
          c.modality = a;
          c.max_rows = c.rows_static = (int32_t)P->n_mod[a];
          c.qrow0_static = (a == MSA_VIDEO) ? (int32_t)round_up(P->n_mod[0], TILE) : 0;
          if (two) {
            c.k_src = SRC_K2D;
            c.kc_lo = 0;
            c.kc_hi = (int32_t)P->n_mod[a];
            c.krow_lo = (int32_t)region0[a];
            int64_t xv = 0;
            for (int b = 0; b < 2; ++b) xv += budget_scale(cfg.k_v, P->n_mod[b], L);
            c.x_cap = (int32_t)round_up(std::max<int64_t>(xv, 1), TILE);
            has2d = true;
          } else {
            c.x_cap = (int32_t)round_up(std::min<int64_t>(cfg.k_v, L), TILE);
          }
          C.push_back(c);
        }
        break;
      }
    }
    H.n_classes = (int32_t)C.size() - H.class0;
    bool perm = false;
    int32_t xr = 0;
    for (int c = H.class0; c < (int)C.size(); ++c) {
      if (C[c].flags & CF_PERMUTED) perm = true;
      C[c].x_row0 = xr;
      xr += C[c].x_cap;
    }
    H.x_rows = xr;
    if (perm) H.q_slice = n_qslices++;
    if (xr > 0) H.x_slice = n_xslices++;
    H.q_rows = perm ? LP : 0;
    x_rows_max = std::max(x_rows_max, xr);
  }
  // ---- work items: grouped by KV head, then key source, then head kind.  The items in flight
  // then read one copy of one head's K and V (which stays in L2 while the group runs, where it
  // fits) and move through it at about the same pace (items of one kind cost about the same per
  // tile), so that they reuse each other's tiles in L2.  Within a group: slots from the last
  // (most keys) to the first with the query heads interleaved, so that the dynamic assignment
  // in the attention kernel hands out the longest items first.
  {
    int32_t max_slots = 0;
    for (auto& c : C) {
      c.n_items = (int32_t)((c.max_rows + TILE - 1) / TILE);
      max_slots = std::max(max_slots, c.n_items);
      const int64_t nunits = (c.kc_hi - c.kc_lo + UNIT - 1) / UNIT;
      c.tile_cap = (int32_t)(c.x_cap / TILE + (nunits + 1) / 2);
    }
    for (int c = 0; c < (int)C.size(); ++c) C[c].item0 = -1;
    // when every head's K and V fit in L2 together (about half of it), the grouping buys no
    // reuse and only delays the last group's longest items: plain longest-first order then
    const bool group = (int64_t)Hkv * L * 512 * (has2d ? 2 : 1) > (64ll << 20);
    if (group) {
      for (int32_t g = 0; g < prob->Hkv; ++g)
        for (int32_t src : {SRC_K, SRC_K2D})  // K/V in original order, then the modality-grouped copy
          for (int32_t kind = MSA_DENSE; kind <= MSA_BOUND2D; ++kind)
            for (int32_t s = max_slots - 1; s >= 0; --s)
              for (int c = 0; c < (int)C.size(); ++c)
                if (C[c].kvh == g && C[c].k_src == src && prob->heads[C[c].head].kind == kind && s < C[c].n_items)
                  P->items.push_back(WorkItem{c, s});
    } else {
      for (int32_t s = max_slots - 1; s >= 0; --s)
        for (int c = 0; c < (int)C.size(); ++c)
          if (s < C[c].n_items) P->items.push_back(WorkItem{c, s});
    }
    // ---- key chunks of the attention kernel: when one head's K and V (L x 512 B) no longer fit
    // comfortably in L2, the keys are cut into 128K-key chunks (64 MB of K and V per head); the
    // environment variable MSA_ATTN_CHUNK_KEYS (a multiple of 128) overrides the chunk size.
    int64_t ck = (int64_t)L * 512 > (96ll << 20) ? 131072 : 0;
    if (const char* env = std::getenv("MSA_ATTN_CHUNK_KEYS")) ck = std::max<int64_t>(0, std::atoll(env)) / TILE * TILE;
    P->n_kchunks = (ck > 0 && ck < L) ? (int32_t)((L + ck - 1) / ck) : 1;
    P->chunk_keys = P->n_kchunks > 1 ? (int32_t)ck : (int32_t)L;
    P->bands.clear();
    P->band_cap = 0;
    if (P->n_kchunks > 1) {
      // bands: runs of the plan order within one (KV head, key source, head kind) group and one
      // range of 1024 slots, merged until each holds at least 2048 units.  Alternate bands use
      // two accumulator buffers; a unit of band b writes its item's slot only after every unit
      // of band b - 2 (the previous user of the buffer) has finished (a per-band completion
      // counter that the attention kernel waits on), so the two buffers are safe whatever the
      // order in which the units complete.  The band size only decides how often that wait can
      // stall.  MSA_ATTN_BAND_SLOTS and MSA_ATTN_MIN_BAND_UNITS (read here) override the two
      // sizes, so that tests can make the bands tiny.
      int32_t BAND_SLOTS = 1024, MIN_UNITS = 2048;
      if (const char* env = std::getenv("MSA_ATTN_BAND_SLOTS")) BAND_SLOTS = std::max(1, std::atoi(env));
      if (const char* env = std::getenv("MSA_ATTN_MIN_BAND_UNITS")) MIN_UNITS = std::max(1, std::atoi(env));
      auto key = [&](const WorkItem& w) {
        const ClassStatic& c = C[w.cls];
        return std::make_tuple(c.kvh, c.k_src, prob->heads[c.head].kind, w.slot / BAND_SLOTS);
      };
      int32_t i0 = 0;
      const int32_t n = (int32_t)P->items.size();
      int64_t unit0 = 0;
      for (int32_t i = 1; i <= n; ++i) {
        const bool cut = i == n || key(P->items[i]) != key(P->items[i - 1]);
        if (!cut) continue;
        if (i < n && (int64_t)(i - i0) * P->n_kchunks < MIN_UNITS) continue;  // merge into the next run
        UnitBand b{i0, i - i0, 0, (int32_t)unit0};
        P->bands.push_back(b);
        unit0 += (int64_t)b.n * P->n_kchunks;
        P->band_cap = std::max(P->band_cap, b.n);
        i0 = i;
      }
      for (size_t b = 0; b < P->bands.size(); ++b) P->bands[b].acc0 = (int32_t)(b & 1) * P->band_cap;
      if (unit0 > INT32_MAX) {
        delete P;
        return MSA_ERR_UNSUPPORTED;
      }
      P->n_units = (int32_t)unit0;
    } else {
      P->n_units = (int32_t)P->items.size();
    }
    int64_t tb = 0;
    for (auto& c : C) {
      c.tile_base = tb;
      tb += (int64_t)c.n_items * c.tile_cap;
    }
    P->total_tiles = tb;
    for (int c = 0; c < (int)C.size(); ++c) C[c].dyn = c;
  }
  // ---- estimation row sets and top-k jobs
  std::vector<RowSet>& RS = P->rowsets;
  for (int32_t h = 0; h < Hq; ++h) {
    const msa_head_cfg& cfg = P->heads[h];
    // a_rows: modality of the rows (-1: any); seg >= 0: rows of that segment only
    auto add = [&](int a_rows, int k_src, int32_t a_rank, int seg = -1) -> int {
      RowSet r{};
      r.head = h;
      r.kvh = h / G;
      r.k_src = k_src;
      r.cls = -1;
      std::vector<int32_t> rows;
      if (seg >= 0) {
        const msa_segment& sg = P->segs[seg];
        for (int64_t t = std::max<int64_t>(sg.start, sg.start + sg.len - LASTQ); t < sg.start + sg.len; ++t)
          rows.push_back((int32_t)t);
      } else {
        rows = last_rows(*P, a_rows);
      }
      r.n_rows = (int32_t)rows.size();
      int32_t lo = INT32_MAX, hi = INT32_MIN;
      for (int i = 0; i < r.n_rows; ++i) {
        r.rows[i] = rows[i];
        r.rcs[i] = (a_rank >= 0) ? (int32_t)(region0[a_rank] + P->rank[rows[i]]) : rows[i];
        lo = std::min(lo, r.rcs[i]);
        hi = std::max(hi, r.rcs[i]);
      }
      r.span = r.n_rows ? hi - lo : 0;
      r.key_hi = (k_src == SRC_K2D) ? (int32_t)L : (r.n_rows ? rows.back() + 1 : 0);
      RS.push_back(r);
      return (int)RS.size() - 1;
    };
    switch (cfg.kind) {
      case MSA_VSLASH: {
        int i = add(-1, SRC_K, -1);
        RS[i].slash_lo = 0;
        RS[i].slash_hi = (int32_t)L;
        break;
      }
      case MSA_GRID: {
        int i = add(MSA_VIDEO, SRC_K, -1);
        RS[i].slash_lo = RS[i].slash_hi = 0;
        break;
      }
      case MSA_QBOUND:
        if (cfg.flags & MSA_HEAD_PER_SEGMENT) {
          // the last 64 queries of every segment, feeding that segment's class
          for (int c = HS[h].class0; c < HS[h].class0 + HS[h].n_classes; ++c) {
            int i = add(C[c].modality, SRC_K, -1, C[c].seg);
            RS[i].slash_lo = 0;
            RS[i].slash_hi = (int32_t)L;
            RS[i].cls = c;
          }
          break;
        }
        for (int a = 0; a < 2; ++a) {
          if (P->n_mod[a] == 0) continue;
          int i = add(a, SRC_K, -1);
          RS[i].slash_lo = 0;
          RS[i].slash_hi = (int32_t)L;
        }
        break;
      case MSA_BOUND2D:
        for (int a = 0; a < 2; ++a) {
          if (P->n_mod[a] == 0) continue;
          int i = add(a, SRC_K2D, a);
          RS[i].slash_lo = (int32_t)region0[a];
          RS[i].slash_hi = (int32_t)(region0[a] + P->n_mod[a]);
        }
        break;
      default: break;
    }
  }
  // Tiles of the last-query sweep: row sets of one KV head and key source, paired in the order
  // they were made (a head's own row sets first), two per 128-row tensor-core tile.
  std::vector<LqTile>& LT = P->lqtiles;
  LT.clear();
  {
    std::vector<bool> used(RS.size(), false);
    for (size_t i = 0; i < RS.size(); ++i) {
      if (used[i]) continue;
      used[i] = true;
      LqTile t{};
      t.rs[0] = (int32_t)i;
      t.rs[1] = -1;
      t.kvh = RS[i].kvh;
      t.k_src = RS[i].k_src;
      for (size_t j = i + 1; j < RS.size(); ++j)
        if (!used[j] && RS[j].kvh == t.kvh && RS[j].k_src == t.k_src) {
          used[j] = true;
          t.rs[1] = (int32_t)j;
          break;
        }
      LT.push_back(t);
    }
  }
  // key chunks of the sweep (one CTA per tile and chunk)
  std::vector<int32_t> tile_hi;
  for (const auto& t : LT)
    tile_hi.push_back(t.rs[1] >= 0 ? std::max(RS[t.rs[0]].key_hi, RS[t.rs[1]].key_hi) : RS[t.rs[0]].key_hi);
  const int32_t chunk = lastq_pick_chunk(tile_hi.data(), (int)tile_hi.size());
  int32_t max_span = 0;
  for (auto& r : RS) {
    if (r.span > 4096) {
      delete P;
      return MSA_ERR_UNSUPPORTED;
    }
    r.chunk = chunk;
    r.n_chunks = (int32_t)((r.key_hi + r.chunk - 1) / r.chunk);
    if (r.slash_hi > r.slash_lo) max_span = std::max(max_span, r.span);
  }
  for (auto& t : LT) {
    t.key_hi = RS[t.rs[0]].key_hi;
    t.n_chunks = RS[t.rs[0]].n_chunks;
    if (t.rs[1] >= 0) {
      t.key_hi = std::max(t.key_hi, RS[t.rs[1]].key_hi);
      t.n_chunks = std::max(t.n_chunks, RS[t.rs[1]].n_chunks);
    }
  }
  const int32_t lq_ring = lastq_ring_entries(max_span);

  // ---- layout
  lay.header = B.take(256);
  lay.classes = B.take((int64_t)sizeof(ClassStatic) * C.size());
  lay.heads = B.take((int64_t)sizeof(HeadStatic) * Hq);
  lay.rowsets = B.take((int64_t)sizeof(RowSet) * RS.size());
  lay.lq_tiles = B.take((int64_t)sizeof(LqTile) * std::max<size_t>(LT.size(), 1));
  // jobs are sized below (after raw slots exist); reserve the maximum: 2 + 4 per row set
  const int64_t max_jobs = (int64_t)RS.size() * 3 + 1;
  lay.jobs = B.take((int64_t)sizeof(TopkJob) * max_jobs);
  lay.items = B.take((int64_t)sizeof(WorkItem) * P->items.size());
  lay.bands = B.take((int64_t)sizeof(UnitBand) * std::max<size_t>(P->bands.size(), 1));
  lay.segs = B.take(4 * (int64_t)P->segtab.size());
  P->blob_bytes = B.off;
  lay.class_dyn = B.take((int64_t)sizeof(ClassDyn) * C.size());
  lay.item_ntiles = B.take(4 * (int64_t)P->items.size());
  if (P->n_kchunks > 1) {
    lay.cstart = B.take(4 * (int64_t)P->items.size() * (P->n_kchunks + 1));
    // chunk_done: uint32 [n_items] followed by the per-band completion counters [n_bands]
    lay.chunk_done = B.take(4 * ((int64_t)P->items.size() + (int64_t)P->bands.size()));
    lay.acc = B.take(4 * 2 * (int64_t)P->band_cap * TILE * ACC_ROW, 1024);
  }
  lay.tiles = B.take(4 * P->total_tiles);
  lay.mask_pairs = B.take(8 * (int64_t)Hq);
  lay.modality = B.take(L);
  lay.rank = B.take(4 * L);
  lay.perm2d = B.take(4 * L);
  lay.mod_rows[0] = lay.perm2d;
  lay.mod_rows[1] = lay.perm2d + 4 * region0[1];
  for (int32_t h = 0; h < Hq; ++h) {
    HeadStatic& H = HS[h];
    const msa_head_cfg& cfg = P->heads[h];
    H.counts_off = B.take(64 + 4 * 3 * 32);  // list counts; grid heads: per-block counts of the materialisation
    const bool per_seg = (cfg.flags & MSA_HEAD_PER_SEGMENT) != 0;  // lists live in the classes
    if ((cfg.kind == MSA_VSLASH || cfg.kind == MSA_QBOUND || cfg.kind == MSA_BOUND2D) && !per_seg) {
      for (int a = 0; a < 2; ++a) {
        if (P->n_mod[a] == 0 && cfg.kind != MSA_VSLASH) continue;
        if (cfg.kind == MSA_VSLASH && a > 0) continue;
        for (int b = 0; b < 2; ++b) {
          int32_t cap = 0;
          if (cfg.kind == MSA_BOUND2D) cap = budget_scale(cfg.k_v, P->n_mod[b], L);
          else if (b == 0) cap = (int32_t)std::min<int64_t>(cfg.k_v, L);
          if (cap <= 0) continue;
          H.rawv_cap[a][b] = cap;
          H.rawv_off[a][b] = B.take(4 * (int64_t)cap);
        }
        int32_t cs = cfg.kind == MSA_BOUND2D ? budget_scale(cfg.k_s, P->n_mod[a], L)
                                             : (int32_t)std::min<int64_t>(cfg.k_s, L);
        H.raws_cap[a] = cs;
        H.raws_off[a] = B.take(4 * (int64_t)cs);
      }
    }
    if (cfg.kind == MSA_GRID) {
      int32_t smax = 1;
      for (int i = 0; i < cfg.n_strides; ++i) smax = std::max(smax, cfg.strides[i]);
      H.phases_off = B.take(4 * (int64_t)smax);
    }
    if (cfg.kind == MSA_BLOCK) {
      int64_t kmax;
      if (cfg.topk_blocks > 0) kmax = std::min<int64_t>(cfg.topk_blocks, nb);
      else kmax = std::min<int64_t>(nb, (int64_t)std::ceil(cfg.block_budget * (double)nb));
      kmax = std::max<int64_t>(kmax, 1);
      H.blk_kmax = (int32_t)kmax;
      H.blk_nb = (int32_t)nb;
      H.blk_fixed = cfg.topk_blocks;
      H.blk_budget = cfg.block_budget;
      H.blk_list_off = B.take(4 * nb * kmax);
      H.blk_cnt_off = B.take(4 * nb);
      H.qbar_off = B.take(4 * nb * D);
    }
  }
  for (auto& c : C) {
    const HeadStatic& H = HS[c.head];
    if (c.flags & CF_DYNROWS) c.rows_off = B.take(4 * L);
    else if (c.flags & CF_SEGIDX)  // the segment's positions: a run of its modality's list
      c.rows_off = lay.mod_rows[c.modality] + 4 * (int64_t)P->rank[P->segs[c.seg].start];
    else if (c.flags & CF_PERMUTED) c.rows_off = lay.mod_rows[c.modality];
    if (c.flags & CF_SEGIDX) {
      c.segv_off = B.take(4 * (int64_t)std::max(c.segv_cap, 1));
      c.segs_off = B.take(4 * (int64_t)std::max(c.segs_cap, 1));
      c.segcnt_off = B.take(8);
    }
    if (c.flags & CF_X) c.x_pos_off = B.take(4 * (int64_t)c.x_cap);
    if (c.flags & CF_SLASH) {
      c.slash_bits_off = B.take(4 * nwords);
      int a = (c.kind == MSA_VSLASH) ? 0 : c.modality;
      c.slash_list_off = (c.flags & CF_SEGIDX) ? c.segs_off : H.raws_off[a];
    }
    if (c.flags & CF_EXCL) c.excl_bits_off = B.take(4 * nwords);
    if (c.flags & CF_BLOCK) c.blk_bits_off = B.take(4 * nb * (int64_t)c.blk_wpr);
  }
  for (auto& r : RS) {
    r.v_off = B.take(4 * L);
    r.s_off = B.take(4 * L);
    r.mz_off = B.take(4 * (int64_t)r.n_chunks * LASTQ * 2);
    r.stat_off = B.take(4 * LASTQ * 2);
  }
  // top-k jobs
  for (auto& r : RS) {
    const msa_head_cfg& cfg = P->heads[r.head];
    const HeadStatic& H = HS[r.head];
    if (cfg.kind == MSA_GRID || r.n_rows == 0) continue;
    const int32_t maxrow = r.rows[r.n_rows - 1];
    int32_t maxrc = r.rcs[0];
    for (int i = 0; i < r.n_rows; ++i) maxrc = std::max(maxrc, r.rcs[i]);
    if (r.cls >= 0) {  // a segment's own lists
      const ClassStatic& c = C[r.cls];
      TopkJob jv{};
      jv.score_off = r.v_off;
      jv.lo = 0;
      jv.hi = maxrow + 1;
      jv.k = c.segv_cap;
      jv.out_off = c.segv_off;
      jv.cnt_off = c.segcnt_off;
      P->jobs.push_back(jv);
      TopkJob js{};
      js.score_off = r.s_off;
      js.lo = 0;
      js.hi = maxrc + 1;
      js.k = c.segs_cap;
      js.out_off = c.segs_off;
      js.cnt_off = c.segcnt_off + 4;
      P->jobs.push_back(js);
      continue;
    }
    if (cfg.kind == MSA_BOUND2D) {
      const int a = P->mod[r.rows[0]];
      for (int b = 0; b < 2; ++b) {
        if (H.rawv_cap[a][b] <= 0) continue;
        int64_t cnt = 0;  // keys of modality b at positions <= maxrow: a prefix of region b
        for (int64_t t = 0; t <= maxrow; ++t) cnt += (P->mod[t] == b);
        TopkJob j{};
        j.score_off = r.v_off;
        j.lo = (int32_t)region0[b];
        j.hi = (int32_t)(region0[b] + cnt);
        j.k = H.rawv_cap[a][b];
        j.map_k2d = 1;
        j.out_off = H.rawv_off[a][b];
        j.cnt_off = H.counts_off + 4 * (a * 2 + b);
        P->jobs.push_back(j);
      }
      TopkJob j{};
      j.score_off = r.s_off;
      j.lo = 0;
      j.hi = maxrc - (int32_t)region0[a] + 1;
      j.k = H.raws_cap[a];
      j.out_off = H.raws_off[a];
      j.cnt_off = H.counts_off + 4 * (4 + a);
      P->jobs.push_back(j);
    } else {
      const int a = (cfg.kind == MSA_QBOUND) ? P->mod[r.rows[0]] : 0;
      TopkJob jv{};
      jv.score_off = r.v_off;
      jv.lo = 0;
      jv.hi = maxrow + 1;
      jv.k = H.rawv_cap[a][0];
      jv.out_off = H.rawv_off[a][0];
      jv.cnt_off = H.counts_off + 4 * (a * 2);
      P->jobs.push_back(jv);
      TopkJob js{};
      js.score_off = r.s_off;
      js.lo = 0;
      js.hi = maxrc + 1;
      js.k = H.raws_cap[a];
      js.out_off = H.raws_off[a];
      js.cnt_off = H.counts_off + 4 * (4 + a);
      P->jobs.push_back(js);
    }
  }
  if ((int64_t)P->jobs.size() > max_jobs) {
    delete P;
    return MSA_ERR_INVALID_ARG;
  }
  lay.kbar = has_block ? B.take(4 * (int64_t)Hkv * nb * D) : 0;
  lay.xk = B.take(2 * (int64_t)std::max(n_xslices, 1) * std::max(x_rows_max, TILE) * D, 1024);
  lay.xv = B.take(2 * (int64_t)std::max(n_xslices, 1) * std::max(x_rows_max, TILE) * D, 1024);
  lay.k2d = has2d ? B.take(2 * (int64_t)Hkv * L * D, 1024) : 0;
  lay.v2d = has2d ? B.take(2 * (int64_t)Hkv * L * D, 1024) : 0;
  lay.indexed_total = round_up(B.off, 256);
  // the permuted Q and O copies come last: the index-based prefill does without them
  lay.qp = B.take(2 * (int64_t)std::max(n_qslices, 1) * LP * D, 1024);
  lay.op = B.take(2 * (int64_t)Hq * LP * D, 1024);
  lay.total = round_up(B.off, 256);

  // ---- the blob uploaded into the workspace at every estimate / set_indices
  P->blob.assign(P->blob_bytes, 0);
  std::memcpy(P->blob.data() + lay.classes, C.data(), sizeof(ClassStatic) * C.size());
  std::memcpy(P->blob.data() + lay.heads, HS.data(), sizeof(HeadStatic) * Hq);
  if (!RS.empty()) std::memcpy(P->blob.data() + lay.rowsets, RS.data(), sizeof(RowSet) * RS.size());
  if (!LT.empty()) std::memcpy(P->blob.data() + lay.lq_tiles, LT.data(), sizeof(LqTile) * LT.size());
  if (!P->jobs.empty()) std::memcpy(P->blob.data() + lay.jobs, P->jobs.data(), sizeof(TopkJob) * P->jobs.size());
  std::memcpy(P->blob.data() + lay.items, P->items.data(), sizeof(WorkItem) * P->items.size());
  if (!P->bands.empty()) std::memcpy(P->blob.data() + lay.bands, P->bands.data(), sizeof(UnitBand) * P->bands.size());
  std::memcpy(P->blob.data() + lay.segs, P->segtab.data(), 4 * P->segtab.size());

  DevPlan& dp = P->dp;
  dp.ws = nullptr;
  dp.lay = lay;
  dp.L = L;
  dp.Hq = Hq;
  dp.Hkv = Hkv;
  dp.LP = LP;
  dp.n_classes = (int32_t)C.size();
  dp.n_heads = Hq;
  dp.n_rowsets = (int32_t)RS.size();
  dp.n_jobs = (int32_t)P->jobs.size();
  dp.n_items = (int32_t)P->items.size();
  dp.n_units = P->n_units;
  dp.n_kchunks = P->n_kchunks;
  dp.chunk_keys = P->chunk_keys;
  dp.n_bands = (int32_t)P->bands.size();
  dp.n_segs = (int32_t)P->segs.size();
  dp.x_rows = std::max(x_rows_max, TILE);
  dp.n_qslices = n_qslices;
  dp.n_xslices = n_xslices;
  dp.has2d = has2d;
  dp.has_block = has_block;
  dp.n_block_heads = 0;
  for (int32_t h = 0; h < Hq; ++h) dp.n_block_heads += prob->heads[h].kind == MSA_BLOCK ? 1 : 0;
  dp.nb = (int32_t)nb;
  dp.n_text = P->n_mod[0];
  dp.scale = P->scale;
  int32_t tbw = 1, mc = 1;
  P->class_kind.clear();
  for (const auto& c : C) {
    const int64_t nunits = (c.kc_hi - c.kc_lo + UNIT - 1) / UNIT;
    tbw = std::max<int32_t>(tbw, (int32_t)((nunits + 31) / 32 + 1));
    P->class_kind.push_back(c.kind);
  }
  for (const auto& r : RS) mc = std::max(mc, r.n_chunks);
  dp.tb_words = tbw;
  dp.max_chunks = mc;
  dp.n_lqtiles = (int32_t)LT.size();
  dp.lq_ring = lq_ring;
  dp.class_kind = P->class_kind.data();
  *out = P;
  return MSA_OK;
}

void msa_plan_destroy(msa_plan* plan) { delete plan; }

size_t msa_workspace_bytes(const msa_plan* plan) { return plan ? (size_t)plan->lay.total : 0; }

size_t msa_workspace_bytes_indexed(const msa_plan* plan) { return plan ? (size_t)plan->lay.indexed_total : 0; }

}  // extern "C"

// ------------------------------------------------------------------------------------------
namespace {

msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// `full`: the call uses the permuted Q / O copies (msa_permute, msa_sparse_prefill,
// msa_unpermute); the others need only the indexed part of the layout.
msa_status check_ws(const msa_plan* P, const void* ws, size_t bytes, bool full) {
  if (!P || !ws) return MSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256) return MSA_ERR_ALIGN;
  if (bytes < (size_t)(full ? P->lay.total : P->lay.indexed_total)) return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

msa_status check_tensor(const void* p, int64_t sh, int64_t sr) {
  if (!p) return MSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) % 16) return MSA_ERR_ALIGN;
  if (sh % 8 || sr % 8 || sr < D || sh < 0) return MSA_ERR_ALIGN;
  return MSA_OK;
}

DevPlan dev(const msa_plan* P, void* ws) {
  DevPlan d = P->dp;
  d.ws = static_cast<uint8_t*>(ws);
  return d;
}

msa_status upload(msa_plan* P, void* ws, cudaStream_t st) {
  cudaError_t e = cudaMemcpyAsync(ws, P->blob.data(), P->blob_bytes, cudaMemcpyHostToDevice, st);
  return cuda_status(e);
}

}  // namespace

extern "C" {

msa_status msa_estimate(msa_plan* P, const void* Q, const void* K, const msa_strides* s, void* ws, size_t ws_bytes,
                        void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, false);
  if (st != MSA_OK) return st;
  if (!s) return MSA_ERR_INVALID_ARG;
  if ((st = check_tensor(Q, s->q_head, s->q_row)) != MSA_OK) return st;
  if ((st = check_tensor(K, s->k_head, s->k_row)) != MSA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if ((st = upload(P, ws, cs)) != MSA_OK) return st;
  DevPlan d = dev(P, ws);
  cudaError_t e = launch_layout(d, cs);
  if (e == cudaSuccess && d.n_rowsets > 0) e = launch_lastq(d, Q, K, *s, cs);
  if (e == cudaSuccess && d.n_jobs > 0) e = launch_topk_jobs(d, cs);
  if (e == cudaSuccess && d.has_block) e = launch_block_estimate(d, Q, K, *s, cs);
  if (e == cudaSuccess) e = launch_grid_detect(d, cs);
  if (e == cudaSuccess) e = launch_materialize(d, cs);
  if (e == cudaSuccess) e = launch_tiles(d, cs);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  P->ready_ws = ws;
  return MSA_OK;
}

msa_status msa_set_indices(msa_plan* P, const msa_head_indices* heads, void* ws, size_t ws_bytes, void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, false);
  if (st != MSA_OK) return st;
  if (!heads) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // validate and stage every list into one host buffer laid out like the workspace slots
  std::vector<std::pair<int64_t, std::vector<int32_t>>> puts;
  const int64_t L = P->L, nb = L / BLK;
  for (int32_t h = 0; h < P->Hq; ++h) {
    const HeadStatic& H = P->hs[h];
    const msa_head_indices& x = heads[h];
    std::vector<int32_t> counts(8, 0);
    auto sorted_in = [&](const int32_t* v, int32_t n, int64_t lo, int64_t hi) -> bool {
      if (n < 0 || (n > 0 && !v)) return false;
      for (int32_t i = 0; i < n; ++i) {
        if (v[i] < lo || v[i] >= hi) return false;
        if (i && v[i] <= v[i - 1]) return false;
      }
      return true;
    };
    if (P->heads[h].flags & MSA_HEAD_PER_SEGMENT) {  // one pair of lists per segment
      if (x.n_seg != (int32_t)P->segs.size() || !x.seg_nv || !x.seg_v || !x.seg_ns || !x.seg_s)
        return MSA_ERR_INVALID_ARG;
      for (int c = H.class0; c < H.class0 + H.n_classes; ++c) {
        const ClassStatic& cl = P->classes[c];
        const int k = cl.seg;
        const int32_t nv = x.seg_nv[k], ns = x.seg_ns[k];
        if (nv > cl.segv_cap || !sorted_in(x.seg_v[k], nv, 0, L)) return MSA_ERR_INVALID_ARG;
        if (ns > cl.segs_cap || !sorted_in(x.seg_s[k], ns, 0, L)) return MSA_ERR_INVALID_ARG;
        puts.emplace_back(cl.segv_off, std::vector<int32_t>(x.seg_v[k], x.seg_v[k] + nv));
        puts.emplace_back(cl.segs_off, std::vector<int32_t>(x.seg_s[k], x.seg_s[k] + ns));
        puts.emplace_back(cl.segcnt_off, std::vector<int32_t>{nv, ns});
      }
      puts.emplace_back(H.counts_off, counts);
      continue;
    }
    switch (H.kind) {
      case MSA_VSLASH:
      case MSA_QBOUND:
      case MSA_BOUND2D:
        for (int a = 0; a < 2; ++a) {
          for (int b = 0; b < 2; ++b) {
            if (H.rawv_cap[a][b] <= 0) continue;
            const int32_t n = x.n_v[a][b];
            if (n > H.rawv_cap[a][b] || !sorted_in(x.v[a][b], n, 0, L)) return MSA_ERR_INVALID_ARG;
            for (int32_t i = 0; i < n; ++i) {
              if (H.kind == MSA_BOUND2D && P->mod[x.v[a][b][i]] != b) return MSA_ERR_INVALID_ARG;
            }
            counts[a * 2 + b] = n;
            puts.emplace_back(H.rawv_off[a][b], std::vector<int32_t>(x.v[a][b], x.v[a][b] + n));
          }
          if (H.raws_cap[a] > 0) {
            const int32_t n = x.n_s[a];
            if (n > H.raws_cap[a] || !sorted_in(x.s[a], n, 0, L)) return MSA_ERR_INVALID_ARG;
            counts[4 + a] = n;
            puts.emplace_back(H.raws_off[a], std::vector<int32_t>(x.s[a], x.s[a] + n));
          }
        }
        break;
      case MSA_GRID: {
        int np_max = -1;
        for (int i = 0; i < H.grid_n_cand; ++i)
          if (H.grid_cand[i] == x.stride) np_max = H.grid_np[i];
        if (np_max < 0 || x.n_phases < 0 || x.n_phases > np_max || !sorted_in(x.phases, x.n_phases, 0, x.stride))
          return MSA_ERR_INVALID_ARG;
        counts[6] = x.stride;
        counts[7] = x.n_phases;
        puts.emplace_back(H.phases_off, std::vector<int32_t>(x.phases, x.phases + x.n_phases));
        break;
      }
      case MSA_BLOCK: {
        if (!x.blk_ptr || !x.blk_idx) return MSA_ERR_INVALID_ARG;
        std::vector<int32_t> lists((size_t)nb * H.blk_kmax, 0), cnt(nb, 0);
        for (int64_t b = 0; b < nb; ++b) {
          const int32_t n = x.blk_ptr[b + 1] - x.blk_ptr[b];
          if (n < 0 || n > H.blk_kmax || !sorted_in(x.blk_idx + x.blk_ptr[b], n, 0, b + 1))
            return MSA_ERR_INVALID_ARG;
          cnt[b] = n;
          std::copy(x.blk_idx + x.blk_ptr[b], x.blk_idx + x.blk_ptr[b + 1], lists.begin() + b * H.blk_kmax);
        }
        puts.emplace_back(H.blk_list_off, std::move(lists));
        puts.emplace_back(H.blk_cnt_off, std::move(cnt));
        break;
      }
      default: break;
    }
    puts.emplace_back(H.counts_off, counts);
  }
  if ((st = upload(P, ws, cs)) != MSA_OK) return st;
  for (auto& pr : puts) {
    if (pr.second.empty()) continue;
    cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(ws) + pr.first, pr.second.data(), 4 * pr.second.size(),
                                    cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    // pageable sources: the copy is staged before cudaMemcpyAsync returns
  }
  DevPlan d = dev(P, ws);
  cudaError_t e = launch_layout(d, cs);
  if (e == cudaSuccess) e = launch_materialize(d, cs);
  if (e == cudaSuccess) e = launch_tiles(d, cs);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  P->ready_ws = ws;
  return MSA_OK;
}

msa_status msa_permute(msa_plan* P, const void* Q, const void* K, const void* V, const msa_strides* s, void* ws,
                       size_t ws_bytes, void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, true);
  if (st != MSA_OK) return st;
  if (!s) return MSA_ERR_INVALID_ARG;
  if ((st = check_tensor(Q, s->q_head, s->q_row)) != MSA_OK) return st;
  if ((st = check_tensor(K, s->k_head, s->k_row)) != MSA_OK) return st;
  if ((st = check_tensor(V, s->v_head, s->v_row)) != MSA_OK) return st;
  if (P->ready_ws != ws) return MSA_ERR_STATE;
  return cuda_status(launch_permute(dev(P, ws), Q, K, V, *s, true, static_cast<cudaStream_t>(stream)));
}

msa_status msa_sparse_prefill(msa_plan* P, const void* Q, const void* K, const void* V, const msa_strides* s,
                              void* ws, size_t ws_bytes, float* lse, void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, true);
  if (st != MSA_OK) return st;
  if (!s) return MSA_ERR_INVALID_ARG;
  if ((st = check_tensor(Q, s->q_head, s->q_row)) != MSA_OK) return st;
  if ((st = check_tensor(K, s->k_head, s->k_row)) != MSA_OK) return st;
  if ((st = check_tensor(V, s->v_head, s->v_row)) != MSA_OK) return st;
  if (lse && reinterpret_cast<uintptr_t>(lse) % 4) return MSA_ERR_ALIGN;
  if (P->ready_ws != ws) return MSA_ERR_STATE;
  return cuda_status(launch_attention(dev(P, ws), Q, K, V, *s, lse, nullptr, static_cast<cudaStream_t>(stream)));
}

msa_status msa_sparse_prefill_indexed(msa_plan* P, const void* Q, const void* K, const void* V, void* O,
                                      const msa_strides* s, void* ws, size_t ws_bytes, float* lse, void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, false);
  if (st != MSA_OK) return st;
  if (!s) return MSA_ERR_INVALID_ARG;
  if ((st = check_tensor(Q, s->q_head, s->q_row)) != MSA_OK) return st;
  if ((st = check_tensor(K, s->k_head, s->k_row)) != MSA_OK) return st;
  if ((st = check_tensor(V, s->v_head, s->v_row)) != MSA_OK) return st;
  if ((st = check_tensor(O, s->o_head, s->o_row)) != MSA_OK) return st;
  if (lse && reinterpret_cast<uintptr_t>(lse) % 4) return MSA_ERR_ALIGN;
  if (P->ready_ws != ws) return MSA_ERR_STATE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const DevPlan d = dev(P, ws);
  cudaError_t e = launch_permute(d, Q, K, V, *s, false, cs);  // key gathers only
  if (e == cudaSuccess) e = launch_attention(d, Q, K, V, *s, lse, O, cs);
  return cuda_status(e);
}

msa_status msa_unpermute(msa_plan* P, const void* ws, size_t ws_bytes, void* O, const msa_strides* s, void* stream) {
  msa_status st = check_ws(P, ws, ws_bytes, true);
  if (st != MSA_OK) return st;
  if (!s) return MSA_ERR_INVALID_ARG;
  if ((st = check_tensor(O, s->o_head, s->o_row)) != MSA_OK) return st;
  if (P->ready_ws != ws) return MSA_ERR_STATE;
  return cuda_status(launch_unpermute(dev(P, const_cast<void*>(ws)), O, *s, static_cast<cudaStream_t>(stream)));
}

msa_status msa_device_status(const msa_plan* P, void* ws, void* stream) {
  if (!P || !ws) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t err = 0;
  uint8_t* hdr = static_cast<uint8_t*>(ws) + P->lay.header;
  if (cudaMemcpyAsync(&err, hdr, 4, cudaMemcpyDeviceToHost, cs) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  if (err) {
    uint32_t zero = 0;
    if (cudaMemcpy(hdr, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess) return MSA_ERR_CUDA;
  }
  if (err & DEV_ERR_TIMEOUT) return MSA_ERR_TIMEOUT;
  if (err & DEV_ERR_BOUNDS) return MSA_ERR_DEVICE_BOUNDS;
  return MSA_OK;
}

msa_status msa_attention_units(const msa_plan* P, int64_t out[3]) {
  if (!P || !out) return MSA_ERR_INVALID_ARG;
  out[0] = P->n_units;
  out[1] = P->n_kchunks;
  out[2] = (int64_t)P->bands.size();
  return MSA_OK;
}

msa_status msa_tile_stats(const msa_plan* P, const void* ws, int64_t tiles[2], void* stream) {
  if (!P || !ws || !tiles) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  std::vector<int32_t> nt(P->items.size());
  if (cudaMemcpyAsync(nt.data(), static_cast<const uint8_t*>(ws) + P->lay.item_ntiles, 4 * nt.size(),
                      cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  int64_t t = 0, n = 0;
  for (int32_t x : nt) {
    if (x > 0) {
      t += x;
      ++n;
    }
  }
  tiles[0] = t;
  tiles[1] = n;
  return MSA_OK;
}

msa_status msa_tile_stats_heads(const msa_plan* P, const void* ws, int64_t* tiles, void* stream) {
  if (!P || !ws || !tiles) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  std::vector<int32_t> nt(P->items.size());
  if (cudaMemcpyAsync(nt.data(), static_cast<const uint8_t*>(ws) + P->lay.item_ntiles, 4 * nt.size(),
                      cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  for (int32_t h = 0; h < P->Hq; ++h) tiles[h] = 0;
  for (size_t i = 0; i < nt.size(); ++i)
    if (nt[i] > 0) tiles[P->classes[P->items[i].cls].head] += nt[i];
  return MSA_OK;
}

msa_status msa_selftest_timeout(const msa_plan* P, void* ws, uint32_t limit_us, void* stream) {
  if (!P || !ws || limit_us == 0 || limit_us > 1000000u) return MSA_ERR_INVALID_ARG;
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + P->lay.header);
  return cuda_status(launch_wait_probe(status, (uint64_t)limit_us * 1000ull, static_cast<cudaStream_t>(stream)));
}

msa_status msa_mask_pairs(const msa_plan* P, void* ws, int64_t* counts, void* stream) {
  if (!P || !ws || !counts) return MSA_ERR_INVALID_ARG;
  if (P->ready_ws != ws) return MSA_ERR_STATE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = launch_mask_count(dev(P, ws), cs)) return cuda_status(e);
  std::vector<uint64_t> c(P->Hq);
  if (cudaMemcpyAsync(c.data(), static_cast<const uint8_t*>(ws) + P->lay.mask_pairs, 8 * c.size(),
                      cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  for (int32_t h = 0; h < P->Hq; ++h) counts[h] = (int64_t)c[h];
  return MSA_OK;
}

msa_status msa_read_indices(const msa_plan* P, const void* ws, int32_t head, int32_t* out, int64_t* len,
                            void* stream) {
  if (!P || !ws || !len || head < 0 || head >= P->Hq) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const HeadStatic& H = P->hs[head];
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  auto fetch = [&](int64_t off, int64_t n) -> std::vector<int32_t> {
    std::vector<int32_t> v(std::max<int64_t>(n, 0));
    if (n > 0) cudaMemcpyAsync(v.data(), w + off, 4 * n, cudaMemcpyDeviceToHost, cs);
    return v;
  };
  std::vector<int32_t> counts = fetch(H.counts_off, 8);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  std::vector<int32_t> rec;
  rec.push_back(H.kind);
  if (H.kind == MSA_GRID) {
    int32_t np = counts[7];
    std::vector<int32_t> ph = fetch(H.phases_off, np);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
    rec.push_back(counts[6]);
    rec.push_back(np);
    rec.insert(rec.end(), ph.begin(), ph.end());
  } else {
    rec.push_back(0);
    rec.push_back(0);
  }
  for (int a = 0; a < 2; ++a)
    for (int b = 0; b < 2; ++b) {
      int32_t n = H.rawv_cap[a][b] > 0 ? counts[a * 2 + b] : 0;
      std::vector<int32_t> v = fetch(H.rawv_off[a][b], n);
      if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
      rec.push_back(n);
      rec.insert(rec.end(), v.begin(), v.end());
    }
  for (int a = 0; a < 2; ++a) {
    int32_t n = H.raws_cap[a] > 0 ? counts[4 + a] : 0;
    std::vector<int32_t> v = fetch(H.raws_off[a], n);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
    rec.push_back(n);
    rec.insert(rec.end(), v.begin(), v.end());
  }
  if (H.kind == MSA_BLOCK) {
    const int64_t nb = H.blk_nb;
    std::vector<int32_t> cnt = fetch(H.blk_cnt_off, nb);
    std::vector<int32_t> lists = fetch(H.blk_list_off, nb * H.blk_kmax);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
    rec.push_back((int32_t)nb);
    int32_t acc = 0;
    rec.push_back(0);
    for (int64_t b = 0; b < nb; ++b) rec.push_back(acc += cnt[b]);
    for (int64_t b = 0; b < nb; ++b)
      rec.insert(rec.end(), lists.begin() + b * H.blk_kmax, lists.begin() + b * H.blk_kmax + cnt[b]);
  } else {
    rec.push_back(0);
  }
  if (P->heads[head].flags & MSA_HEAD_PER_SEGMENT) {  // the lists of every segment, in order
    rec.push_back(H.n_classes);
    for (int c = H.class0; c < H.class0 + H.n_classes; ++c) {
      const ClassStatic& cl = P->classes[c];
      std::vector<int32_t> cnt = fetch(cl.segcnt_off, 2);
      if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
      const int32_t nv = std::min(std::max(cnt[0], 0), cl.segv_cap), ns = std::min(std::max(cnt[1], 0), cl.segs_cap);
      std::vector<int32_t> v = fetch(cl.segv_off, nv), sl = fetch(cl.segs_off, ns);
      if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
      rec.push_back(nv);
      rec.insert(rec.end(), v.begin(), v.end());
      rec.push_back(ns);
      rec.insert(rec.end(), sl.begin(), sl.end());
    }
  } else {
    rec.push_back(0);
  }
  const int64_t need = (int64_t)rec.size();
  if (!out || *len < need) {
    *len = need;
    return MSA_ERR_INVALID_ARG;
  }
  std::copy(rec.begin(), rec.end(), out);
  *len = need;
  return MSA_OK;
}

msa_status msa_read_tiles(const msa_plan* P, const void* ws, int32_t head, int32_t* out, int64_t* len,
                          void* stream) {
  if (!P || !ws || !len || head < 0 || head >= P->Hq) return MSA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  const int64_t L = P->L;
  std::vector<ClassDyn> dyn(P->classes.size());
  std::vector<int32_t> ntiles(P->items.size()), perm2d(L);
  cudaMemcpyAsync(dyn.data(), w + P->lay.class_dyn, sizeof(ClassDyn) * dyn.size(), cudaMemcpyDeviceToHost, cs);
  cudaMemcpyAsync(ntiles.data(), w + P->lay.item_ntiles, 4 * ntiles.size(), cudaMemcpyDeviceToHost, cs);
  cudaMemcpyAsync(perm2d.data(), w + P->lay.perm2d, 4 * L, cudaMemcpyDeviceToHost, cs);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  std::vector<int32_t> rec;
  rec.push_back(0);
  int32_t n_items = 0;
  for (size_t i = 0; i < P->items.size(); ++i) {
    const WorkItem& wi = P->items[i];
    const ClassStatic& c = P->classes[wi.cls];
    if (c.head != head) continue;
    const ClassDyn& cd = dyn[c.dyn];
    const int32_t nrows = (c.flags & CF_DYNROWS) ? cd.nrows : c.rows_static;
    const int32_t row0 = wi.slot * TILE;
    if (row0 >= nrows) continue;
    std::vector<int32_t> rows(TILE, -1);
    if (c.flags & CF_PERMUTED) {
      const int32_t n = std::min(TILE, nrows - row0);
      cudaMemcpyAsync(rows.data(), w + c.rows_off + 4 * (int64_t)row0, 4 * n, cudaMemcpyDeviceToHost, cs);
    } else {
      for (int t = 0; t < TILE; ++t) rows[t] = (row0 + t < nrows) ? row0 + t : -1;
    }
    const int32_t nt = ntiles[i];
    std::vector<uint32_t> tl(std::max(nt, 0));
    if (nt > 0)
      cudaMemcpyAsync(tl.data(), w + P->lay.tiles + 4 * (c.tile_base + (int64_t)wi.slot * c.tile_cap), 4 * nt,
                      cudaMemcpyDeviceToHost, cs);
    std::vector<int32_t> xpos;
    if ((c.flags & CF_X) && cd.x_len > 0) {
      xpos.resize(c.x_cap);
      cudaMemcpyAsync(xpos.data(), w + c.x_pos_off, 4 * (int64_t)c.x_cap, cudaMemcpyDeviceToHost, cs);
    }
    std::vector<uint32_t> excl;
    if (c.flags & CF_EXCL) {
      excl.resize((L + 31) / 32);
      cudaMemcpyAsync(excl.data(), w + c.excl_bits_off, 4 * excl.size(), cudaMemcpyDeviceToHost, cs);
    }
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
    rec.push_back(wi.cls);
    rec.push_back(std::max(0, std::min(TILE, nrows - row0)));
    rec.insert(rec.end(), rows.begin(), rows.end());
    rec.push_back(nt);
    for (int32_t k = 0; k < nt; ++k) {
      const int src = (int)(tl[k] >> 28);
      const int32_t row = (int32_t)(tl[k] & TILE_ROW_MASK);
      rec.push_back(src | ((tl[k] & TILE_FULL) ? 8 : 0));
      for (int cc = 0; cc < TILE; ++cc) {
        int32_t pos = -1;
        if (src == SRC_X) {
          int32_t idx = row - c.x_row0 + cc;
          if (idx >= 0 && idx < cd.x_len && idx < (int32_t)xpos.size()) pos = xpos[idx];
        } else {
          int64_t coord = (int64_t)c.kc_lo + (row - c.krow_lo) + cc;
          const bool excluded = !excl.empty() && coord >= 0 && coord < L && ((excl[coord >> 5] >> (coord & 31)) & 1u);
          if (coord >= c.kc_lo && coord < c.kc_hi && !excluded) {
            int64_t r = (int64_t)row + cc;
            pos = (src == SRC_K2D) ? perm2d[r] : (int32_t)r;
          }
        }
        rec.push_back(pos);
      }
    }
    ++n_items;
  }
  rec[0] = n_items;
  const int64_t need = (int64_t)rec.size();
  if (!out || *len < need) {
    *len = need;
    return MSA_ERR_INVALID_ARG;
  }
  std::copy(rec.begin(), rec.end(), out);
  *len = need;
  return MSA_OK;
}

}  // extern "C"
