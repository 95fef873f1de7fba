// Host layer of libkvc: layout validation, closed-form buffer sizes, split
// planning and the C ABI entry points declared in include/kvc.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <string>

#include "kvc_internal.h"

struct kvc_layout {
  kvc_layout_desc d;
  int G, L, ngk, ngv;
  int lk_row, lv_row, lksz_row, lvsz_row;  // bytes per row
  int64_t rows;                             // rows per low-rank component
  int qdim, vdim;
  int units;                                // independent (row, head) units of the split kernel
  size_t sizes[KVC_NBUF];
  float scale;
};

namespace {

thread_local std::string g_err;
thread_local int g_test_no_copies = 0;   // kvc_test_skip_tile_copies
thread_local int g_rope_kernel = 0;      // kvc_select_rope_kernel
thread_local int g_varrate_kernel = 0;   // 0: lane-per-head warp kernel, 1: tensor-core kernel

kvc_status fail(kvc_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

kvc_status ok() {
  g_err.clear();
  return KVC_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Bytes of one VARRATE record per KV head at rank r (codes + (scale, zero) pairs).
int varrate_head_bytes(int r) { return r / 2 + 4 * ceil_div(r, 32); }

// Split planning: S splits per unit so that units * S covers about two waves
// of the 148 SMs, each split a whole number of tiles.
void plan(const kvc_layout* L, int n_tokens, int* S, int* split_len) {
  const int tile = kvc::split_tile(L->d.kind, L->d.rope);
  const int tiles = n_tokens > 0 ? ceil_div(n_tokens, tile) : 1;
  int s = ceil_div(2 * kvc::kNumSMs, L->units > 0 ? L->units : 1);
  if (s < 1) s = 1;
  if (s > tiles) s = tiles;
  int per = ceil_div(tiles, s);
  *split_len = per * tile;
  *S = ceil_div(tiles, per);
}

// Workspace: a 256-byte header (error word), the projected queries, then the
// split partials; sized for the larger of the two split plans.
constexpr size_t kWsHeader = 256;

int fast_slots(const kvc_layout* L, int n_tokens) {
  if (n_tokens <= 0) return 1;
  const int tpu = ceil_div(n_tokens, 128);
  const int total = L->d.batch * L->d.n_kv_heads * tpu;
  int g = total < kvc::kNumSMs ? total : kvc::kNumSMs;
  const int w = ceil_div(total, g);
  return (ceil_div(tpu, w) + 1) * kvc::kRopeTcParts;
}

size_t ws_bytes(const kvc_layout* L, int n_tokens) {
  int S, len;
  plan(L, n_tokens, &S, &len);
  const int nt1 = n_tokens > 0 ? n_tokens : 1;
  const int Sf = L->d.kind == KVC_DENSE_BF16
                     ? kvc::dense_tc_slots(L->d.batch, L->d.n_kv_heads, nt1)
                     : fast_slots(L, n_tokens);
  if (Sf > S) S = Sf;
  if (L->d.kind == KVC_LOWRANK) {
    const int Sl = kvc::latent_tc_slots(L->d.batch, L->d.n_kv_heads, nt1);
    if (Sl > S) S = Sl;
    const int Sr = kvc::rope_mma_slots(L->d.batch, L->d.n_kv_heads, nt1);
    if (Sr > S) S = Sr;
    const int Sw = kvc::rope_wg_slots(L->d.batch, L->d.n_kv_heads, nt1);
    if (Sw > S) S = Sw;
  }
  if (L->d.kind == KVC_VARRATE) {
    const int Sv = kvc::varrate_warp_slots(L->d.batch, nt1);
    if (Sv > S) S = Sv;
  }
  if (L->d.kind == KVC_BLOCK_SHARED) {
    const int Sb = kvc::block_mma_slots(L->d.batch, L->L, L->d.n_q_heads, nt1);
    if (Sb > S) S = Sb;
    const int St = kvc::block_tc_slots(L->d.batch, nt1);
    if (St > S) S = St;
  }
  const size_t rows = (size_t)L->L * L->d.batch * L->d.n_q_heads;
  size_t b = kWsHeader + round_up(rows * L->qdim * sizeof(float), 256);
  b += round_up((size_t)S * rows * (L->vdim + 2) * sizeof(float), 256);
  return b;
}

}  // namespace

kvc_status kvc::report_error(kvc_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

extern "C" {

const char* kvc_last_error(void) { return g_err.c_str(); }

void kvc_test_skip_tile_copies(int32_t on) { g_test_no_copies = on ? 1 : 0; }

void kvc_select_rope_kernel(int32_t which) { g_rope_kernel = which == 2 ? 2 : 0; }

void kvc_select_varrate_kernel(int32_t which) { g_varrate_kernel = which == 1 ? 1 : 0; }

const char* kvc_version(void) {
  return "kvc 0.3 (sm_100a; decode kernels rev 16; rope_mma rev 13)";
}

kvc_status kvc_create_layout(const kvc_layout_desc* desc, kvc_layout** out) {
  if (!desc || !out) return fail(KVC_EINVAL, "kvc_create_layout: NULL argument");
  *out = nullptr;
  kvc_layout_desc d = *desc;
  if (d.n_layers <= 0) d.n_layers = 1;
  if (d.kind < KVC_DENSE_BF16 || d.kind > KVC_VARRATE)
    return fail(KVC_EINVAL, "unknown kind %d", d.kind);
  if (d.batch < 1 || d.batch > kvc::kMaxBatch)
    return fail(KVC_EINVAL, "batch %d outside 1..%d", d.batch, kvc::kMaxBatch);
  if (d.n_kv_heads < 1 || d.n_q_heads < 1 || d.n_q_heads % d.n_kv_heads)
    return fail(KVC_EINVAL, "n_q_heads %d must be a positive multiple of n_kv_heads %d",
                d.n_q_heads, d.n_kv_heads);
  if (d.head_dim != 64 && d.head_dim != 128)
    return fail(KVC_EUNSUPPORTED, "head_dim %d (64 or 128 supported)", d.head_dim);
  if (d.max_tokens < 1) return fail(KVC_EINVAL, "max_tokens %d", d.max_tokens);
  if (d.rope && d.kind != KVC_LOWRANK)
    return fail(KVC_EUNSUPPORTED, "rope is a LOWRANK option");
  if (d.rope && !(d.rope_theta > 1.0)) return fail(KVC_EINVAL, "rope_theta must be > 1");
  if (d.resid_bits != 0 && d.resid_bits != 2)
    return fail(KVC_EUNSUPPORTED, "resid_bits %d (0 or 2)", d.resid_bits);
  if (d.resid_bits && (d.kind != KVC_LOWRANK || d.head_dim != kvc::kResidDim))
    return fail(KVC_EUNSUPPORTED, "a rotated residual needs LOWRANK with head_dim 128");
  if (d.page_size != 0 && d.page_size != 16)
    return fail(KVC_EUNSUPPORTED, "page_size %d (0 or 16)", d.page_size);
  if (d.page_size && d.kind != KVC_LOWRANK)
    return fail(KVC_EUNSUPPORTED, "paging is a LOWRANK option");
  if (d.page_size && (d.max_tokens % d.page_size || d.n_pages < 1))
    return fail(KVC_EINVAL, "paged: max_tokens %% page_size must be 0 and n_pages >= 1");
  if (d.n_layers > 1 && d.kind != KVC_BLOCK_SHARED && d.kind != KVC_DENSE_BF16)
    return fail(KVC_EUNSUPPORTED, "n_layers > 1 only for BLOCK_SHARED and DENSE");

  kvc_layout* L = new (std::nothrow) kvc_layout();
  if (!L) return fail(KVC_EINVAL, "out of host memory");
  L->d = d;
  L->G = d.n_q_heads / d.n_kv_heads;
  L->L = d.n_layers;
  L->scale = d.softmax_scale > 0 ? d.softmax_scale : 1.0f / sqrtf((float)d.head_dim);
  memset(L->sizes, 0, sizeof(L->sizes));
  const size_t B = d.batch, Hkv = d.n_kv_heads, T = d.max_tokens, hd = d.head_dim;
  kvc_status st = KVC_OK;
  const char* why = "";

  switch (d.kind) {
    case KVC_LOWRANK: {
      if (d.rank_k < 2 || d.rank_v < 2 || d.rank_k % 2 || d.rank_v % 2 || d.rank_k > 128 ||
          d.rank_v > 128) {
        st = KVC_EINVAL, why = "ranks must be even in 2..128";
        break;
      }
      if (d.latent_bits != 16 && d.latent_bits != 4) {
        st = KVC_EUNSUPPORTED, why = "latent_bits must be 16 or 4";
        break;
      }
      if (d.latent_bits == 4 && (d.group_size < 2 || d.group_size % 2)) {
        st = KVC_EINVAL, why = "group_size must be even and >= 2";
        break;
      }
      if (d.latent_bits == 16 && d.resid_bits) {
        st = KVC_EUNSUPPORTED, why = "a residual needs an INT4 latent";
        break;
      }
      L->rows = d.page_size ? (int64_t)d.n_pages * Hkv * d.page_size : (int64_t)B * Hkv * T;
      if (d.latent_bits == 4) {
        L->ngk = ceil_div(d.rank_k, d.group_size);
        L->ngv = ceil_div(d.rank_v, d.group_size);
        L->lk_row = d.rank_k / 2;
        L->lv_row = d.rank_v / 2;
        L->lksz_row = 4 * L->ngk;
        L->lvsz_row = 4 * L->ngv;
      } else {
        L->lk_row = 2 * d.rank_k;
        L->lv_row = 2 * d.rank_v;
      }
      L->sizes[KVC_BUF_LK_CODES] = (size_t)L->rows * L->lk_row;
      L->sizes[KVC_BUF_LV_CODES] = (size_t)L->rows * L->lv_row;
      L->sizes[KVC_BUF_LK_SZ] = (size_t)L->rows * L->lksz_row;
      L->sizes[KVC_BUF_LV_SZ] = (size_t)L->rows * L->lvsz_row;
      if (d.resid_bits) {
        L->sizes[KVC_BUF_RK_CODES] = L->sizes[KVC_BUF_RV_CODES] = (size_t)L->rows * hd / 4;
        L->sizes[KVC_BUF_RK_SCALE] = L->sizes[KVC_BUF_RV_SCALE] = (size_t)L->rows * 2;
        L->sizes[KVC_BUF_SIGNS_K] = L->sizes[KVC_BUF_SIGNS_V] = hd;
      }
      L->sizes[KVC_BUF_BK] = Hkv * d.rank_k * hd * 2;
      L->sizes[KVC_BUF_BV] = Hkv * d.rank_v * hd * 2;
      if (d.page_size) L->sizes[KVC_BUF_PAGE_TABLE] = B * (T / d.page_size) * 4;
      const int res = d.resid_bits ? kvc::kResidDim : 0;
      L->qdim = d.rope ? 0 : d.rank_k + res;
      L->vdim = d.rank_v + res;
      L->units = (int)(B * Hkv);
      break;
    }
    case KVC_VARRATE: {
      if (d.rank_k != 64 || d.rank_v != 64 || d.latent_bits != 4 || d.group_size != 32) {
        st = KVC_EUNSUPPORTED, why = "VARRATE needs rank_k = rank_v = 64, latent_bits 4, group 32";
        break;
      }
      const size_t per_tok = Hkv * varrate_head_bytes(64);
      L->sizes[KVC_BUF_LK_CODES] = L->sizes[KVC_BUF_LV_CODES] = B * T * per_tok;
      L->sizes[KVC_BUF_OFFSET_K] = L->sizes[KVC_BUF_OFFSET_V] = B * (T + 1) * 4;
      L->sizes[KVC_BUF_RANK_K] = L->sizes[KVC_BUF_RANK_V] = B * T;
      L->sizes[KVC_BUF_BK] = L->sizes[KVC_BUF_BV] = Hkv * 64 * hd * 2;
      L->qdim = 64;
      L->vdim = 64;
      L->units = (int)(B * Hkv);
      break;
    }
    case KVC_BLOCK_SHARED: {
      // the decode kernels hold the 32 queries' accumulators of a CTA in
      // registers (at most 64 per thread): latent widths up to 512
      if (d.latent_dim < 16 || d.latent_dim > 512 || d.latent_dim % 16) {
        st = KVC_EINVAL, why = "latent_dim must be a multiple of 16 in 16..512";
        break;
      }
      if (d.group_size < 2 || d.latent_dim % d.group_size || d.group_size % 2) {
        st = KVC_EINVAL, why = "group_size must be even and divide latent_dim";
        break;
      }
      if (d.latent_dim / d.group_size > 64) {
        st = KVC_EUNSUPPORTED, why = "at most 64 scale groups per latent";
        break;
      }
      if ((d.n_layers * d.n_q_heads) % kvc::kBlockQueries) {
        st = KVC_EUNSUPPORTED, why = "n_layers * n_q_heads must be a multiple of 32";
        break;
      }
      if (d.latent_bits == 0) d.latent_bits = 4;
      if (d.latent_bits != 3 && d.latent_bits != 4 && d.latent_bits != 8) {
        st = KVC_EUNSUPPORTED, why = "block-shared latent_bits must be 3, 4 or 8";
        break;
      }
      if (d.value_bits != 0 && d.value_bits != 2 && d.value_bits != 3 && d.value_bits != 4 &&
          d.value_bits != 8) {
        st = KVC_EUNSUPPORTED, why = "value_bits must be 0 (shared latent) or 2, 3, 4, 8";
        break;
      }
      L->d.latent_bits = d.latent_bits;
      const size_t ngs = d.latent_dim / d.group_size;
      L->sizes[KVC_BUF_LK_CODES] = B * T * d.latent_dim * d.latent_bits / 8;
      L->sizes[KVC_BUF_LK_SZ] = B * T * ngs * 2;
      if (d.value_bits) {
        L->sizes[KVC_BUF_LV_CODES] = B * T * d.latent_dim * d.value_bits / 8;
        L->sizes[KVC_BUF_LV_SZ] = B * T * ngs * 2;
      }
      L->sizes[KVC_BUF_BK] = L->sizes[KVC_BUF_BV] =
          (size_t)d.n_layers * d.latent_dim * Hkv * hd * 2;
      L->qdim = d.latent_dim;
      L->vdim = d.latent_dim;
      L->units = (int)(B * d.n_layers * d.n_q_heads / kvc::kBlockQueries);
      break;
    }
    case KVC_DENSE_BF16: {
      L->sizes[KVC_BUF_K_DENSE] = L->sizes[KVC_BUF_V_DENSE] =
          (size_t)d.n_layers * B * Hkv * T * hd * 2;
      L->qdim = 0;
      L->vdim = d.head_dim;
      L->units = (int)(d.n_layers * B * Hkv);
      break;
    }
  }
  if (st != KVC_OK) {
    delete L;
    return fail(st, "kvc_create_layout: %s", why);
  }
  *out = L;
  return ok();
}

void kvc_destroy_layout(kvc_layout* layout) { delete layout; }

kvc_status kvc_buffer_sizes(const kvc_layout* L, size_t sizes[KVC_NBUF]) {
  if (!L || !sizes) return fail(KVC_EINVAL, "kvc_buffer_sizes: NULL argument");
  memcpy(sizes, L->sizes, sizeof(L->sizes));
  return ok();
}

size_t kvc_step_bytes(const kvc_layout* L, int32_t n) {
  if (!L || n <= 0) return 0;
  const kvc_layout_desc& d = L->d;
  const size_t rowsB = (size_t)d.batch * d.n_kv_heads * n;
  switch (d.kind) {
    case KVC_LOWRANK: {
      size_t per = L->lk_row + L->lv_row + L->lksz_row + L->lvsz_row;
      if (d.resid_bits) per += 2 * (d.head_dim / 4 + 2);
      return rowsB * per;
    }
    case KVC_VARRATE: {
      // expected record bytes under the rank mix {4,8,16,32,64} x {.4,.25,.2,.1,.05}
      const double ef = 0.4 * 6 + 0.25 * 8 + 0.2 * 12 + 0.1 * 20 + 0.05 * 40;
      return (size_t)((double)rowsB * 2 * ef) + (size_t)d.batch * n * 10;
    }
    case KVC_BLOCK_SHARED: {
      const size_t scales = 2 * (d.latent_dim / d.group_size);
      size_t per = d.latent_dim * d.latent_bits / 8 + scales;
      if (d.value_bits) per += d.latent_dim * d.value_bits / 8 + scales;
      return (size_t)d.batch * n * per;
    }
    case KVC_DENSE_BF16:
      return (size_t)d.n_layers * rowsB * d.head_dim * 2 * 2;
  }
  return 0;
}

size_t kvc_workspace_bytes(const kvc_layout* L, int32_t n_tokens) {
  if (!L) return 0;
  return ws_bytes(L, n_tokens < 0 ? 0 : n_tokens);
}

int32_t kvc_decode_launches(const kvc_layout* L, int32_t n_tokens) {
  if (!L) return 0;
  kvc::Params p = {};
  p.kind = L->d.kind;
  p.rope = L->d.rope;
  // uniform lengths: the variable-rate layout of 8 KV heads x 4 query heads
  // runs the warp kernel, which projects its own queries
  if (p.kind == KVC_VARRATE && L->d.n_kv_heads == 8 && L->d.n_q_heads == 32 &&
      L->d.group_size == 32 && n_tokens > 0)
    p.path = g_varrate_kernel ? 9 : 5;
  return 2 + (kvc::needs_qproj(p) ? 1 : 0);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// parameter assembly shared by append and decode
// ----------------------------------------------------------------------------

static kvc_status fill_params(const kvc_layout* L, const kvc_cache* c, kvc::Params* p) {
  const kvc_layout_desc& d = L->d;
  memset(p, 0, sizeof(*p));
  p->kind = d.kind;
  p->B = d.batch;
  p->Hq = d.n_q_heads;
  p->Hkv = d.n_kv_heads;
  p->G = L->G;
  p->d = d.head_dim;
  p->L = L->L;
  p->rk = d.rank_k;
  p->rv = d.rank_v;
  p->bits = d.latent_bits;
  p->vbits = d.kind == KVC_BLOCK_SHARED ? d.value_bits : 0;
  p->g = d.group_size;
  p->ngk = L->ngk;
  p->ngv = L->ngv;
  p->resid = d.resid_bits;
  p->rope = d.rope;
  p->page = d.page_size;
  p->tmax = d.max_tokens;
  p->n_pages = d.n_pages;
  p->D = d.latent_dim;
  p->n_tokens = c->n_tokens;
  p->seq_lens = c->seq_lens;
  p->lk_row = L->lk_row;
  p->lv_row = L->lv_row;
  p->lksz_row = L->lksz_row;
  p->lvsz_row = L->lvsz_row;
  p->lk = (const uint8_t*)c->lk_codes;
  p->lksz = (const __half*)c->lk_sz;
  p->lv = (const uint8_t*)c->lv_codes;
  p->lvsz = (const __half*)c->lv_sz;
  p->rkc = (const uint8_t*)c->rk_codes;
  p->rks = (const __half*)c->rk_scale;
  p->rvc = (const uint8_t*)c->rv_codes;
  p->rvs = (const __half*)c->rv_scale;
  p->kd = (const __nv_bfloat16*)c->k_dense;
  p->vd = (const __nv_bfloat16*)c->v_dense;
  p->bk = (const __half*)c->bk;
  p->bv = (const __half*)c->bv;
  p->signs_k = c->signs_k;
  p->signs_v = c->signs_v;
  p->page_table = c->page_table;
  p->off_k = c->offset_k;
  p->off_v = c->offset_v;
  p->rank_k = c->rank_k;
  p->rank_v = c->rank_v;
  p->stream_bytes = d.kind == KVC_VARRATE ? L->sizes[KVC_BUF_LK_CODES] / d.batch : 0;
  p->scale = L->scale;
  p->scale_log2 = L->scale * 1.4426950408889634f;
  p->qdim = L->qdim;
  p->vdim = L->vdim;
  if (d.rope) {
    for (int i = 0; i < d.head_dim / 2; ++i)
      p->rope_f[i] = pow(d.rope_theta, -2.0 * i / d.head_dim) / (2.0 * M_PI);
  }
  // required buffers, by kind
  struct Need { const void* ptr; const char* name; };
  Need need[24];
  int nn = 0;
  switch (d.kind) {
    case KVC_LOWRANK:
      need[nn++] = {c->lk_codes, "lk_codes"};
      need[nn++] = {c->lv_codes, "lv_codes"};
      need[nn++] = {c->bk, "bk"};
      need[nn++] = {c->bv, "bv"};
      if (d.latent_bits == 4) {
        need[nn++] = {c->lk_sz, "lk_sz"};
        need[nn++] = {c->lv_sz, "lv_sz"};
      }
      if (d.resid_bits) {
        need[nn++] = {c->rk_codes, "rk_codes"};
        need[nn++] = {c->rv_codes, "rv_codes"};
        need[nn++] = {c->rk_scale, "rk_scale"};
        need[nn++] = {c->rv_scale, "rv_scale"};
        need[nn++] = {c->signs_k, "signs_k"};
        need[nn++] = {c->signs_v, "signs_v"};
      }
      if (d.page_size) need[nn++] = {c->page_table, "page_table"};
      break;
    case KVC_VARRATE:
      need[nn++] = {c->lk_codes, "lk_codes"};
      need[nn++] = {c->lv_codes, "lv_codes"};
      need[nn++] = {c->offset_k, "offset_k"};
      need[nn++] = {c->offset_v, "offset_v"};
      need[nn++] = {c->rank_k, "rank_k"};
      need[nn++] = {c->rank_v, "rank_v"};
      need[nn++] = {c->bk, "bk"};
      need[nn++] = {c->bv, "bv"};
      break;
    case KVC_BLOCK_SHARED:
      need[nn++] = {c->lk_codes, "lk_codes"};
      need[nn++] = {c->lk_sz, "lk_sz"};
      if (d.value_bits) {
        need[nn++] = {c->lv_codes, "lv_codes (value latent)"};
        need[nn++] = {c->lv_sz, "lv_sz (value latent)"};
      }
      need[nn++] = {c->bk, "bk (W_k)"};
      need[nn++] = {c->bv, "bv (W_v)"};
      break;
    case KVC_DENSE_BF16:
      need[nn++] = {c->k_dense, "k_dense"};
      need[nn++] = {c->v_dense, "v_dense"};
      break;
  }
  for (int i = 0; i < nn; ++i) {
    if (!need[i].ptr) return fail(KVC_EINVAL, "cache.%s is NULL", need[i].name);
    if (!aligned16(need[i].ptr))
      return fail(KVC_EALIGN, "cache.%s is not 16-byte aligned", need[i].name);
  }
  if (c->seq_lens && !aligned16(c->seq_lens))
    return fail(KVC_EALIGN, "cache.seq_lens is not 16-byte aligned");
  return KVC_OK;
}

static kvc_status launch_status(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(KVC_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return KVC_OK;
}

extern "C" kvc_status kvc_decode_attn_timed(const kvc_layout* L, const kvc_cache* c,
                                            const void* q, void* out, void* workspace,
                                            size_t ws_size, void* stream, void* ev_begin,
                                            void* ev_end) {
  if (!L || !c || !q || !out) return fail(KVC_EINVAL, "kvc_decode_attn: NULL argument");
  if (c->n_tokens < 0) return fail(KVC_EINVAL, "n_tokens %d < 0", c->n_tokens);
  if (c->n_tokens > L->d.max_tokens)
    return fail(KVC_ECAPACITY, "n_tokens %d > max_tokens %d", c->n_tokens, L->d.max_tokens);
  if (!aligned16(q) || !aligned16(out))
    return fail(KVC_EALIGN, "q / out must be 16-byte aligned");
  const size_t need = ws_bytes(L, c->n_tokens);
  if (!workspace || ws_size < need)
    return fail(KVC_EWORKSPACE, "workspace %zu bytes < %zu needed", ws_size, need);
  if (!aligned16(workspace)) return fail(KVC_EALIGN, "workspace must be 16-byte aligned");
  kvc::Params p;
  kvc_status st = fill_params(L, c, &p);
  if (st != KVC_OK) return st;
  if (c->layer < 0 || c->layer > L->L)
    return fail(KVC_EINVAL, "cache.layer %d outside 0..%d", c->layer, L->L);
  if (c->layer > 0 && L->L > 1) {
    // one layer of the block: the shared cache with that layer's projections
    // (block-shared) or that layer's slice of the dense cache
    const size_t lo = (size_t)(c->layer - 1);
    if (L->d.kind == KVC_BLOCK_SHARED) {
      const size_t wsz = (size_t)L->d.latent_dim * L->d.n_kv_heads * L->d.head_dim;
      p.bk += lo * wsz;
      p.bv += lo * wsz;
    } else if (L->d.kind == KVC_DENSE_BF16) {
      const size_t lsz = (size_t)L->d.batch * L->d.n_kv_heads * L->d.max_tokens * L->d.head_dim;
      p.kd += lo * lsz;
      p.vd += lo * lsz;
    }
    p.L = 1;
  }
  p.q = (const __nv_bfloat16*)q;
  p.test_no_copies = g_test_no_copies;
  p.out = out;
  p.out_bf16 = L->d.out_bf16;
  plan(L, c->n_tokens, &p.S, &p.split_len);
  {
    // the warp- / CTA-level tensor-core kernels run equal contiguous tile
    // ranges (seg_W tiles of the flattened (unit, tile) space per warp or CTA)
    int grid = 0, W = 0, tpu = 0, slots = 0, parts = 1;
    if (kvc::rope_wg_supported(p) && g_rope_kernel == 2) {
      kvc::rope_wg_plan(p, &grid, &W, &tpu, &slots);
      p.path = 7;
      parts = kvc::kRopeWgParts;
    } else if (kvc::rope_mma_supported(p)) {
      kvc::rope_mma_plan(p, &grid, &W, &tpu, &slots);
      p.path = 4;
    } else if (kvc::rope_tc_supported(p)) {
      kvc::rope_tc_plan(p, &grid, &W, &tpu, &slots);
      p.path = 1;
      parts = kvc::kRopeTcParts;
    } else if (kvc::latent_tc_supported(p)) {
      kvc::latent_tc_plan(p, &grid, &W, &tpu, &slots);
      p.path = 3;
    } else if (kvc::dense_tc_supported(p)) {
      kvc::dense_tc_plan(p, &grid, &W, &tpu, &slots);
      p.path = 2;
    }
    if (p.path) {
      p.S = slots;
      p.seg_W = W;
      p.seg_tpu = tpu;
      p.seg_parts = parts;
    } else if (kvc::varrate_mma_supported(p) && g_varrate_kernel == 1) {
      // fixed token splits per batch row (one partial per CTA)
      kvc::varrate_mma_plan(p, &p.S, &p.split_len);
      p.path = 9;
    } else if (kvc::varrate_warp_supported(p)) {
      kvc::varrate_warp_plan(p, &p.S, &p.split_len);
      p.path = 5;
    } else if (kvc::block_tc_supported(p)) {
      kvc::block_tc_plan(p, &p.S, &p.split_len);
      p.path = 8;
    } else if (kvc::block_mma_supported(p)) {
      kvc::block_mma_plan(p, &p.S, &p.split_len);
      p.path = 6;
    }
  }
  const size_t rows = (size_t)L->L * L->d.batch * L->d.n_q_heads;
  char* ws = (char*)workspace;
  p.err = (uint32_t*)ws;
  p.qt = (float*)(ws + kWsHeader);
  p.part = (float*)(ws + kWsHeader + round_up(rows * L->qdim * sizeof(float), 256));
  cudaStream_t s = (cudaStream_t)stream;
  cudaGetLastError();  // clear a stale error so it is not reported as ours
  if (kvc::path_sets_error_word(p)) {
    // the workspace's previous contents do not matter: start the word at zero
    st = launch_status(cudaMemsetAsync(p.err, 0, sizeof(uint32_t), s), "error word reset");
    if (st != KVC_OK) return st;
  }
  if (kvc::needs_qproj(p)) {
    st = launch_status(kvc::launch_qproj(p, s), "qproj launch");
    if (st != KVC_OK) return st;
  }
  if (ev_begin) cudaEventRecord((cudaEvent_t)ev_begin, s);
  st = launch_status(kvc::launch_split(p, s), "split-T decode launch");
  if (st != KVC_OK) return st;
  if (ev_end) cudaEventRecord((cudaEvent_t)ev_end, s);
  st = launch_status(kvc::launch_combine(p, s), "combine launch");
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" kvc_status kvc_decode_attn(const kvc_layout* L, const kvc_cache* c, const void* q,
                                      void* out, void* workspace, size_t ws_size,
                                      void* stream) {
  return kvc_decode_attn_timed(L, c, q, out, workspace, ws_size, stream, nullptr, nullptr);
}

extern "C" kvc_status kvc_append(const kvc_layout* L, const kvc_cache* c, const void* k_new,
                                 const void* v_new, const int32_t* pos, int32_t n_new,
                                 const uint8_t* new_ranks, void* stream) {
  if (!L || !c || !pos) return fail(KVC_EINVAL, "kvc_append: NULL argument");
  const kvc_layout_desc& d = L->d;
  if (n_new < 1) return fail(KVC_EINVAL, "n_new %d < 1", n_new);
  if (n_new > d.max_tokens)
    return fail(KVC_ECAPACITY, "n_new %d > max_tokens %d", n_new, d.max_tokens);
  if (!k_new || ((d.kind != KVC_BLOCK_SHARED || d.value_bits) && !v_new))
    return fail(KVC_EINVAL, "kvc_append: k_new / v_new is NULL");
  if (!aligned16(k_new) || (v_new && !aligned16(v_new)) || !aligned16(pos))
    return fail(KVC_EALIGN, "k_new / v_new / pos must be 16-byte aligned");
  if (c->status && (reinterpret_cast<uintptr_t>(c->status) & 3u))
    return fail(KVC_EALIGN, "cache.status must be 4-byte aligned");
  if (d.kind == KVC_VARRATE) {
    if (!new_ranks) return fail(KVC_EINVAL, "VARRATE append needs new_ranks");
    if (!aligned16(new_ranks)) return fail(KVC_EALIGN, "new_ranks must be 16-byte aligned");
  }
  kvc::AppendParams* a = new (std::nothrow) kvc::AppendParams();
  if (!a) return fail(KVC_EINVAL, "out of host memory");
  kvc_status st = fill_params(L, c, &a->p);
  if (d.kind == KVC_VARRATE && st == KVC_OK && (!c->offset_k || !c->offset_v))
    st = fail(KVC_EINVAL, "cache offsets are NULL");
  if (st != KVC_OK) {
    delete a;
    return st;
  }
  a->k_new = (const __nv_bfloat16*)k_new;
  a->v_new = (const __nv_bfloat16*)v_new;
  a->n_new = n_new;
  a->pos = pos;
  a->new_ranks = new_ranks;
  a->status = c->status;
  a->lk_w = (uint8_t*)c->lk_codes;
  a->lksz_w = (__half*)c->lk_sz;
  a->lv_w = (uint8_t*)c->lv_codes;
  a->lvsz_w = (__half*)c->lv_sz;
  a->rkc_w = (uint8_t*)c->rk_codes;
  a->rks_w = (__half*)c->rk_scale;
  a->rvc_w = (uint8_t*)c->rv_codes;
  a->rvs_w = (__half*)c->rv_scale;
  a->kd_w = (__nv_bfloat16*)c->k_dense;
  a->vd_w = (__nv_bfloat16*)c->v_dense;
  a->off_k_w = c->offset_k;
  a->off_v_w = c->offset_v;
  a->rank_k_w = c->rank_k;
  a->rank_v_w = c->rank_v;
  cudaStream_t s = (cudaStream_t)stream;
  cudaGetLastError();
  st = launch_status(kvc::launch_append(*a, s), "append launch");
  delete a;
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" size_t kvc_fit_workspace_bytes(int32_t n_kv_heads) {
  return n_kv_heads > 0 ? kvc::fit_workspace_bytes(n_kv_heads) : 0;
}

extern "C" kvc_status kvc_fit_factors(const void* x, int32_t batch, int32_t n_kv_heads,
                                      int32_t capacity, int32_t n_rows, int32_t head_dim,
                                      const float* omega, int32_t k, int32_t rank,
                                      int32_t power_iters, void* factor, float* sigma2,
                                      void* workspace, size_t ws_size, void* stream) {
  if (!x || !omega || !factor || !workspace)
    return fail(KVC_EINVAL, "kvc_fit_factors: NULL argument");
  if (head_dim != 128) return fail(KVC_EUNSUPPORTED, "kvc_fit_factors: head_dim %d (128)", head_dim);
  if (batch < 1 || n_kv_heads < 1 || capacity < 1 || n_rows < 1 || n_rows > capacity)
    return fail(KVC_EINVAL, "kvc_fit_factors: batch %d, heads %d, rows %d of capacity %d", batch,
                n_kv_heads, n_rows, capacity);
  if (k < 2 || k > kvc::kFitMaxK || k % 2 || rank < 1 || rank > k)
    return fail(KVC_EINVAL, "kvc_fit_factors: sketch width %d (even, 2..%d) and rank %d (<= k)",
                k, kvc::kFitMaxK, rank);
  if (power_iters < 0 || power_iters > 16)
    return fail(KVC_EINVAL, "kvc_fit_factors: power_iters %d (0..16)", power_iters);
  if (!aligned16(x) || !aligned16(omega) || !aligned16(factor) || !aligned16(workspace) ||
      (sigma2 && !aligned16(sigma2)))
    return fail(KVC_EALIGN, "kvc_fit_factors: pointers must be 16-byte aligned");
  const size_t need = kvc::fit_workspace_bytes(n_kv_heads);
  if (ws_size < need) return fail(KVC_EWORKSPACE, "workspace %zu bytes < %zu needed", ws_size, need);
  kvc::FitParams f;
  f.x = (const __nv_bfloat16*)x;
  f.B = batch;
  f.Hkv = n_kv_heads;
  f.cap = capacity;
  f.n_rows = n_rows;
  f.omega = omega;
  f.k = k;
  f.rank = rank;
  f.power_iters = power_iters;
  f.factor = (__half*)factor;
  f.sigma2 = sigma2;
  f.workspace = workspace;
  cudaGetLastError();
  kvc_status st = launch_status(kvc::launch_fit(f, (cudaStream_t)stream), "factor fit launch");
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" size_t kvc_salience_workspace_bytes(int32_t batch, int32_t n_q_heads,
                                               int32_t n_kv_heads, int32_t window,
                                               int32_t n_tokens) {
  if (batch < 1 || n_q_heads < 1 || n_kv_heads < 1 || window < 1 || n_tokens < 1) return 0;
  return kvc::salience_workspace_bytes(batch, n_q_heads, n_kv_heads, window, n_tokens);
}

extern "C" kvc_status kvc_window_salience(const void* q_window, const void* keys, int32_t batch,
                                          int32_t n_q_heads, int32_t n_kv_heads, int32_t window,
                                          int32_t capacity, int32_t n_tokens, int32_t head_dim,
                                          float softmax_scale, float* salience, void* workspace,
                                          size_t ws_size, void* stream) {
  if (!q_window || !keys || !salience || !workspace)
    return fail(KVC_EINVAL, "kvc_window_salience: NULL argument");
  if (head_dim != 128) return fail(KVC_EUNSUPPORTED, "kvc_window_salience: head_dim %d (128)", head_dim);
  if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads || window < 1 ||
      n_tokens < 1 || n_tokens > capacity)
    return fail(KVC_EINVAL, "kvc_window_salience: bad sizes");
  if ((n_q_heads / n_kv_heads) * window > kvc::kSalMaxRows)
    return fail(KVC_EUNSUPPORTED, "kvc_window_salience: %d query heads per KV head x window %d > %d",
                n_q_heads / n_kv_heads, window, kvc::kSalMaxRows);
  if (!aligned16(q_window) || !aligned16(keys) || !aligned16(salience) || !aligned16(workspace))
    return fail(KVC_EALIGN, "kvc_window_salience: pointers must be 16-byte aligned");
  const size_t need = kvc::salience_workspace_bytes(batch, n_q_heads, n_kv_heads, window, n_tokens);
  if (ws_size < need) return fail(KVC_EWORKSPACE, "workspace %zu bytes < %zu needed", ws_size, need);
  kvc::SalienceCall c;
  c.q = (const __nv_bfloat16*)q_window;
  c.k = (const __nv_bfloat16*)keys;
  c.B = batch;
  c.Hq = n_q_heads;
  c.Hkv = n_kv_heads;
  c.W = window;
  c.cap = capacity;
  c.T = n_tokens;
  c.scale = softmax_scale > 0 ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  c.sal = salience;
  c.workspace = workspace;
  cudaGetLastError();
  kvc_status st = launch_status(kvc::launch_salience(c, (cudaStream_t)stream), "salience launch");
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" kvc_status kvc_ranks_by_salience(const float* salience, int32_t batch,
                                            int32_t n_tokens, int32_t n_rungs,
                                            const int32_t* rung_ranks, const int32_t* rung_counts,
                                            uint8_t* ranks, void* stream) {
  if (!salience || !rung_ranks || !ranks || (n_rungs > 1 && !rung_counts))
    return fail(KVC_EINVAL, "kvc_ranks_by_salience: NULL argument");
  if (batch < 1 || n_tokens < 1 || n_rungs < 1 || n_rungs > 8)
    return fail(KVC_EINVAL, "kvc_ranks_by_salience: batch %d, tokens %d, rungs %d (1..8)", batch,
                n_tokens, n_rungs);
  kvc::RankLadder lad;
  memset(&lad, 0, sizeof(lad));
  lad.n = n_rungs;
  for (int i = 0; i < n_rungs; ++i) {
    const int r = rung_ranks[i];
    if (r != 4 && r != 8 && r != 16 && r != 32 && r != 64)
      return fail(KVC_EINVAL, "rung %d: rank %d not in {4, 8, 16, 32, 64}", i, r);
    lad.rank[i] = r;
    if (i + 1 < n_rungs) {
      if (rung_counts[i] < 0) return fail(KVC_EINVAL, "rung %d: negative count", i);
      lad.count[i] = rung_counts[i];
    }
  }
  if (!aligned16(salience) || !aligned16(ranks))
    return fail(KVC_EALIGN, "kvc_ranks_by_salience: pointers must be 16-byte aligned");
  cudaGetLastError();
  kvc_status st = launch_status(kvc::launch_ranks(nullptr, 0, const_cast<float*>(salience), batch,
                                                  n_tokens, lad, ranks, (cudaStream_t)stream),
                                "ranks launch");
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" kvc_status kvc_block_keep(const float* salience_layers, int32_t n_layers,
                                     int32_t batch, int32_t n_tokens, int32_t keep,
                                     float* importance, int32_t* kept, void* stream) {
  if (!salience_layers || !importance || !kept)
    return fail(KVC_EINVAL, "kvc_block_keep: NULL argument");
  if (n_layers < 1 || batch < 1 || n_tokens < 1 || keep < 1 || keep > n_tokens)
    return fail(KVC_EINVAL, "kvc_block_keep: layers %d, batch %d, keep %d of %d tokens", n_layers,
                batch, keep, n_tokens);
  if (!aligned16(salience_layers) || !aligned16(importance) || !aligned16(kept))
    return fail(KVC_EALIGN, "kvc_block_keep: pointers must be 16-byte aligned");
  cudaGetLastError();
  kvc_status st = launch_status(kvc::launch_keep(salience_layers, n_layers, importance, batch,
                                                 n_tokens, keep, kept, (cudaStream_t)stream),
                                "keep launch");
  if (st != KVC_OK) return st;
  return ok();
}

extern "C" kvc_status kvc_block_compact(const kvc_layout* src_layout, const kvc_cache* src,
                                        const kvc_layout* dst_layout, const kvc_cache* dst,
                                        const int32_t* kept, int32_t keep, void* stream) {
  if (!src_layout || !src || !dst_layout || !dst || !kept)
    return fail(KVC_EINVAL, "kvc_block_compact: NULL argument");
  const kvc_layout_desc& a = src_layout->d;
  const kvc_layout_desc& b = dst_layout->d;
  if (a.kind != KVC_BLOCK_SHARED || b.kind != KVC_BLOCK_SHARED)
    return fail(KVC_EUNSUPPORTED, "kvc_block_compact: block-shared layouts only");
  if (a.batch != b.batch || a.latent_dim != b.latent_dim || a.group_size != b.group_size)
    return fail(KVC_EINVAL, "kvc_block_compact: the two layouts differ in batch or latent format");
  if (keep < 1 || keep > b.max_tokens || keep > src->n_tokens)
    return fail(KVC_ECAPACITY, "kvc_block_compact: keep %d (source %d tokens, destination holds %d)",
                keep, src->n_tokens, b.max_tokens);
  if (!src->lk_codes || !src->lk_sz || !dst->lk_codes || !dst->lk_sz)
    return fail(KVC_EINVAL, "kvc_block_compact: cache buffers are NULL");
  if (!aligned16(src->lk_codes) || !aligned16(dst->lk_codes) || !aligned16(kept) ||
      !aligned16(src->lk_sz) || !aligned16(dst->lk_sz))
    return fail(KVC_EALIGN, "kvc_block_compact: pointers must be 16-byte aligned");
  cudaGetLastError();
  kvc_status st = launch_status(
      kvc::launch_compact((const uint8_t*)src->lk_codes, (const __half*)src->lk_sz,
                          (uint8_t*)dst->lk_codes, (__half*)dst->lk_sz, kept, a.batch,
                          a.max_tokens, b.max_tokens, keep, a.latent_dim / 2,
                          a.latent_dim / a.group_size, (cudaStream_t)stream),
      "compact launch");
  if (st != KVC_OK) return st;
  return ok();
}
