/*
 * art_oracle.c -- plain, slow CPU oracle for single-token decode attention
 * with ART (runtime attention termination) and the q8 V-dequantisation skip.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Everything is computed in double precision, one (batch, query head) at a
 * time, tile by tile, position by position, in the order the pages describe.
 *
 * Sources (web pages, cited by title and section):
 *   [ART]  "Resumen Tecnico: ART (Terminacion de la Atencion en Tiempo de
 *          Ejecucion)", gist.science summary of arXiv 2606.00024.
 *          S1   decode query attends to the whole cached K/V.
 *          S2.1 tile-wise (FlashAttention style) accumulation; the partial
 *               state after each KV tile is available.
 *          S2.2 probe x^(t) taken from the partial output O^(t); magnitude
 *               change d_scale (difference of L2 norms of x^(t), x^(t-1));
 *               direction change d_direction (deviation of their cosine
 *               similarity); terminate only when both are below their
 *               thresholds (tau, phi) at the same time.
 *          S2.3 patience p: the criterion must hold on p consecutive tiles.
 *          S2.4 block 0 is always evaluated before any termination; tile
 *               order does not change full attention; the traversal order
 *               of the KV blocks may be changed (recency first, importance
 *               first) and ART then watches the probe along that order.
 *   [SKIP] "La paradoja de la eficiencia: como omitir redefine la velocidad
 *          de los LLM", puntofijo.es, section "La Elegancia de la Omision":
 *          the flash kernel knows the softmax weights before it touches V,
 *          so V rows whose weight is negligible need not be dequantised.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - d_scale = | ||x^(t)|| - ||x^(t-1)|| |  (difference of norms).
 *   - d_dir   = max(0, 1 - cos(x^(t), x^(t-1))); 0 when both probes are zero,
 *               1 when exactly one is zero.
 *   - the probe before the first tile of a split is the zero vector.
 *   - "below" is strict (<); a NaN threshold never holds.
 *   - the rule runs per (batch, query head) and independently per KV split
 *     (own tile 0, own history, own patience); tiles = sum over splits.
 *   - split s covers tiles [floor(s*n/S), floor((s+1)*n/S)), n = ceil(L/T).
 *   - a partial last tile counts as one consumed tile.
 *   - V skip (q8 only): row j of the current tile is left out of the
 *     numerator when exp(s_j - m') < tau, m' the running maximum of the
 *     split after the current tile; its weight stays in the denominator.
 *   - q8 value = int8 * (fp16 scale of its 32-element block).
 *   - traversal order (S2.4): an explicit per-(batch, kv head) sequence of
 *     tile indices; the split structure applies to positions in the
 *     sequence, and each split's segment must be a permutation of that
 *     split's own tiles.  Without a sequence the order is 0, 1, ..., n-1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_KV_F32 0
#define ORACLE_KV_BF16 1
#define ORACLE_KV_Q8 2

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_SEQLEN (-2)
#define ORACLE_ERR_NOMEM (-3)

typedef struct {
  int B, Hq, Hkv, d, L_max, tile, num_splits;
} oracle_shape;

typedef struct {
  int enabled;      /* 0: plain attention over every tile */
  double eps_scale; /* tau  (page: magnitude threshold) */
  double eps_dir;   /* phi  (page: direction threshold) */
  int patience;     /* p */
  const int32_t* lanes;
  int n_probe;
} oracle_art;

/* bf16 is the upper half of an IEEE binary32 word. */
double oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 10) & 0x1f;
  int frac = bits & 0x3ff;
  double mag;
  if (expo == 0) {
    mag = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
  } else if (expo == 31) {
    mag = frac ? NAN : INFINITY;
  } else {
    mag = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) * 2^(e-15) */
  }
  return sign ? -mag : mag;
}

/* Decode row `row` (absolute row index into the [B*Hkv*L_max] row space) to doubles. */
static void decode_row(int kind, const void* base, const uint16_t* scales, long row, int d,
                       double* out) {
  if (kind == ORACLE_KV_F32) {
    const float* p = (const float*)base + row * (long)d;
    for (int i = 0; i < d; ++i) out[i] = (double)p[i];
  } else if (kind == ORACLE_KV_BF16) {
    const uint16_t* p = (const uint16_t*)base + row * (long)d;
    for (int i = 0; i < d; ++i) out[i] = oracle_bf16_to_double(p[i]);
  } else {
    const int8_t* p = (const int8_t*)base + row * (long)d;
    const uint16_t* sc = scales + row * (long)(d / 32);
    for (int i = 0; i < d; ++i) out[i] = (double)p[i] * oracle_f16_to_double(sc[i / 32]);
  }
}

/* Running softmax state of one split: running max m, denominator l, numerator acc[d]. */
typedef struct {
  double m, l;
  double* acc;
  int used;
} state_t;

static void state_copy(state_t* dst, const state_t* src, int d) {
  dst->m = src->m;
  dst->l = src->l;
  dst->used = src->used;
  memcpy(dst->acc, src->acc, sizeof(double) * (size_t)d);
}

static double l2norm(const double* x, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += x[i] * x[i];
  return sqrt(s);
}

/*
 * One (batch, query head).  Returns 0 or a negative error.
 * o: [d]; used: [S]; metrics: NULL or [n_tiles_max][2] (d_scale, d_dir) by position in
 * the traversal sequence; seq: NULL (natural order) or this kv head's [n_tiles_max]
 * traversal sequence; vskip: NULL or [L_max], where each row the head weighs with the
 * V skip on gets p / tau (the row left the numerator iff that is below 1).
 */
static int decode_one_head(const oracle_shape* sh, int kind, const void* q, const void* k,
                           const void* v, const uint16_t* k_scale, const uint16_t* v_scale,
                           int L, int b, int hq, const oracle_art* art, double tau,
                           const int32_t* forced_used, int no_break, const int32_t* seq,
                           double* o, int32_t* used, double* metrics, int n_tiles_max, double* vskip) {
  const int d = sh->d, T = sh->tile, S = sh->num_splits;
  const int G = sh->Hq / sh->Hkv;
  const int kvh = hq / G;
  const int n = (L + T - 1) / T;
  const long row0 = ((long)b * sh->Hkv + kvh) * (long)sh->L_max;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  const int P = (art && art->enabled) ? art->n_probe : 0;
  const int skip_on = (kind == ORACLE_KV_Q8) && (tau > 0.0);

  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* kr = (double*)malloc(sizeof(double) * (size_t)d);
  double* vr = (double*)malloc(sizeof(double) * (size_t)d);
  double* sc = (double*)malloc(sizeof(double) * (size_t)T);
  double* x = (double*)malloc(sizeof(double) * (size_t)(P > 0 ? P : 1));
  double* xprev = (double*)malloc(sizeof(double) * (size_t)(P > 0 ? P : 1));
  double* part_m = (double*)malloc(sizeof(double) * (size_t)S);
  double* part_l = (double*)malloc(sizeof(double) * (size_t)S);
  double* part_acc = (double*)calloc((size_t)S * (size_t)d, sizeof(double));
  state_t cur, snap;
  cur.acc = (double*)malloc(sizeof(double) * (size_t)d);
  snap.acc = (double*)malloc(sizeof(double) * (size_t)d);
  if (!qv || !kr || !vr || !sc || !x || !xprev || !part_m || !part_l || !part_acc || !cur.acc ||
      !snap.acc) {
    free(qv); free(kr); free(vr); free(sc); free(x); free(xprev);
    free(part_m); free(part_l); free(part_acc); free(cur.acc); free(snap.acc);
    return ORACLE_ERR_NOMEM;
  }

  /* Q row (q8 mode carries a bf16 query). */
  {
    long qrow = (long)b * sh->Hq + hq;
    if (kind == ORACLE_KV_F32) {
      const float* p = (const float*)q + qrow * d;
      for (int i = 0; i < d; ++i) qv[i] = (double)p[i];
    } else {
      const uint16_t* p = (const uint16_t*)q + qrow * d;
      for (int i = 0; i < d; ++i) qv[i] = oracle_bf16_to_double(p[i]);
    }
  }

  for (int s = 0; s < S; ++s) {
    const int ta = (int)(((long)s * n) / S);
    const int tb = (int)(((long)(s + 1) * n) / S);
    cur.m = -INFINITY;
    cur.l = 0.0;
    cur.used = 0;
    memset(cur.acc, 0, sizeof(double) * (size_t)d);
    for (int i = 0; i < P; ++i) xprev[i] = 0.0;
    int run = 0, stopped = 0;
    const int forced = forced_used ? forced_used[s] : -1;

    for (int kpos = ta; kpos < tb; ++kpos) {
      if (forced >= 0 && cur.used >= forced) break;
      const int t = seq ? seq[kpos] : kpos; /* the tile at this position of the sequence */
      if (t < ta || t >= tb) {
        free(qv); free(kr); free(vr); free(sc); free(x); free(xprev);
        free(part_m); free(part_l); free(part_acc); free(cur.acc); free(snap.acc);
        return ORACLE_ERR_ARG;
      }
      const int j0 = t * T;
      const int j1 = (j0 + T < L) ? j0 + T : L;

      /* S2.1: scores of this tile, and the running max after it. */
      double mt = -INFINITY;
      for (int j = j0; j < j1; ++j) {
        decode_row(kind, k, k_scale, row0 + j, d, kr);
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qv[i] * kr[i];
        sc[j - j0] = dot * inv_sqrt_d;
        if (sc[j - j0] > mt) mt = sc[j - j0];
      }
      const double mnew = (cur.m > mt) ? cur.m : mt;
      const double alpha = (cur.m == -INFINITY) ? 0.0 : exp(cur.m - mnew);
      cur.l *= alpha;
      for (int i = 0; i < d; ++i) cur.acc[i] *= alpha;

      /* Weights of this tile, then V (skipped rows stay in the denominator). */
      for (int j = j0; j < j1; ++j) {
        const double p = exp(sc[j - j0] - mnew);
        cur.l += p;
        if (skip_on && vskip) vskip[j] = p / tau;
        if (skip_on && p < tau) continue;
        decode_row(kind, v, v_scale, row0 + j, d, vr);
        for (int i = 0; i < d; ++i) cur.acc[i] += p * vr[i];
      }
      cur.m = mnew;
      cur.used += 1;

      if (P > 0 && forced < 0) {
        /* S2.2: probe = fixed lanes of the normalised partial output. */
        for (int i = 0; i < P; ++i) x[i] = cur.acc[art->lanes[i]] / cur.l;
        const double a = l2norm(x, P);
        const double bn = l2norm(xprev, P);
        const double d_scale = fabs(a - bn);
        double d_dir;
        if (a == 0.0 && bn == 0.0) {
          d_dir = 0.0;
        } else if (a == 0.0 || bn == 0.0) {
          d_dir = 1.0;
        } else {
          double dot = 0.0;
          for (int i = 0; i < P; ++i) dot += x[i] * xprev[i];
          d_dir = 1.0 - dot / (a * bn);
          if (d_dir < 0.0) d_dir = 0.0;
        }
        if (metrics && kpos < n_tiles_max) {
          metrics[2 * kpos + 0] = d_scale;
          metrics[2 * kpos + 1] = d_dir;
        }
        /* S2.2 + S2.3: both below threshold, on p consecutive tiles. */
        const int hold = (d_scale < art->eps_scale) && (d_dir < art->eps_dir);
        run = hold ? run + 1 : 0;
        for (int i = 0; i < P; ++i) xprev[i] = x[i];
        if (!stopped && run >= art->patience) {
          stopped = 1;
          state_copy(&snap, &cur, d);
          if (!no_break) break;
        }
      }
    }
    if (!stopped) state_copy(&snap, &cur, d);
    part_m[s] = snap.m;
    part_l[s] = snap.l;
    memcpy(part_acc + (size_t)s * d, snap.acc, sizeof(double) * (size_t)d);
    used[s] = snap.used;
  }

  /* Merge the splits: O = sum_s e^{m_s-M} acc_s / sum_s e^{m_s-M} l_s. */
  double M = -INFINITY;
  for (int s = 0; s < S; ++s)
    if (part_m[s] > M) M = part_m[s];
  double den = 0.0;
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  for (int s = 0; s < S; ++s) {
    if (part_m[s] == -INFINITY) continue; /* empty split */
    const double w = exp(part_m[s] - M);
    den += w * part_l[s];
    for (int i = 0; i < d; ++i) o[i] += w * part_acc[(size_t)s * d + i];
  }
  for (int i = 0; i < d; ++i) o[i] /= den;

  free(qv); free(kr); free(vr); free(sc); free(x); free(xprev);
  free(part_m); free(part_l); free(part_acc); free(cur.acc); free(snap.acc);
  return ORACLE_OK;
}

/*
 * Decode every (batch, query head), tiles in the traversal order `tile_order`.
 *   q        f32 [B,Hq,d] for ORACLE_KV_F32, else bf16 bits [B,Hq,d]
 *   k, v     f32 / bf16 bits / int8, [B,Hkv,L_max,d]
 *   k_scale, v_scale  q8 only: fp16 bits [B,Hkv,L_max,d/32]
 *   seq_lens [B], each in [1, L_max]
 *   art      NULL or enabled==0: plain attention
 *   tau      q8 V-skip threshold (<= 0: no skip)
 *   forced_used  NULL or [B,Hq,S]: run each split for exactly that many tiles
 *                (clamped to the split), without the rule
 *   no_break with ART: keep evaluating the rule after the stop so that
 *            metrics cover every tile; outputs still come from the stop tile
 *   o        [B,Hq,d] doubles
 *   used     [B,Hq,S] tiles consumed per split
 *   tiles    [B,Hq] sum of used over splits
 *   metrics  NULL or [B,Hq,n_tiles_max,2] by position in the traversal sequence;
 *            NaN where no rule was evaluated
 *   tile_order  NULL (natural order) or [B,Hkv,n_tiles_max]: the traversal sequence
 *            of each (batch, kv head); entries at positions >= ceil(L_b/T) are ignored
 *   n_threads  OpenMP threads over (batch, query head); <= 0: library default
 *   vskip    NULL or [B,Hq,L_max]: p / tau of every row a head weighed with the q8 V skip
 *            on (p = exp(s_j - m'), m' the running maximum after the row's tile); the row
 *            left that head's numerator iff the value is below 1.  NaN elsewhere.
 * A sequence entry outside its split's tiles gives ORACLE_ERR_ARG.
 */
int oracle_decode_vskip(const oracle_shape* sh, int kind, const void* q, const void* k,
                        const void* v, const uint16_t* k_scale, const uint16_t* v_scale,
                        const int32_t* seq_lens, const oracle_art* art, double tau,
                        const int32_t* forced_used, int no_break, const int32_t* tile_order,
                        double* o, int32_t* used, int32_t* tiles, double* metrics, int n_threads,
                        double* vskip) {
  if (!sh || !q || !k || !v || !seq_lens || !o || !used || !tiles) return ORACLE_ERR_ARG;
  if (sh->B < 1 || sh->Hq < 1 || sh->Hkv < 1 || sh->d < 1 || sh->L_max < 1 || sh->tile < 1 ||
      sh->num_splits < 1)
    return ORACLE_ERR_ARG;
  if (sh->Hq % sh->Hkv != 0) return ORACLE_ERR_ARG;
  if (kind < ORACLE_KV_F32 || kind > ORACLE_KV_Q8) return ORACLE_ERR_ARG;
  if (kind == ORACLE_KV_Q8 && (sh->d % 32 != 0 || !k_scale || !v_scale)) return ORACLE_ERR_ARG;
  if (art && art->enabled) {
    if (art->n_probe < 1 || !art->lanes || art->patience < 1) return ORACLE_ERR_ARG;
    for (int i = 0; i < art->n_probe; ++i)
      if (art->lanes[i] < 0 || art->lanes[i] >= sh->d) return ORACLE_ERR_ARG;
  }
  for (int b = 0; b < sh->B; ++b)
    if (seq_lens[b] < 1 || seq_lens[b] > sh->L_max) return ORACLE_ERR_SEQLEN;

  const int n_tiles_max = (sh->L_max + sh->tile - 1) / sh->tile;
  if (vskip) {
    const long nv = (long)sh->B * sh->Hq * sh->L_max;
    for (long i = 0; i < nv; ++i) vskip[i] = NAN;
  }
  if (metrics) {
    const long nm = (long)sh->B * sh->Hq * n_tiles_max * 2;
    for (long i = 0; i < nm; ++i) metrics[i] = NAN;
  }
  const int S = sh->num_splits;
  const int nheads = sh->B * sh->Hq;
  int err = ORACLE_OK;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(min : err)
#endif
  for (int bh = 0; bh < nheads; ++bh) {
    const int b = bh / sh->Hq, hq = bh % sh->Hq;
    const int kvh = hq / (sh->Hq / sh->Hkv);
    const int32_t* seq = tile_order ? tile_order + ((long)b * sh->Hkv + kvh) * n_tiles_max : NULL;
    int r = decode_one_head(sh, kind, q, k, v, k_scale, v_scale, seq_lens[b], b, hq, art, tau,
                            forced_used ? forced_used + (long)bh * S : NULL, no_break, seq,
                            o + (long)bh * sh->d, used + (long)bh * S,
                            metrics ? metrics + (long)bh * n_tiles_max * 2 : NULL, n_tiles_max,
                            vskip ? vskip + (long)bh * sh->L_max : NULL);
    if (r < err) err = r;
    int sum = 0;
    for (int s = 0; s < S; ++s) sum += used[(long)bh * S + s];
    tiles[bh] = sum;
  }
  return err;
}

/* Without the V-skip record. */
int oracle_decode_ordered(const oracle_shape* sh, int kind, const void* q, const void* k,
                          const void* v, const uint16_t* k_scale, const uint16_t* v_scale,
                          const int32_t* seq_lens, const oracle_art* art, double tau,
                          const int32_t* forced_used, int no_break, const int32_t* tile_order,
                          double* o, int32_t* used, int32_t* tiles, double* metrics,
                          int n_threads) {
  return oracle_decode_vskip(sh, kind, q, k, v, k_scale, v_scale, seq_lens, art, tau, forced_used,
                             no_break, tile_order, o, used, tiles, metrics, n_threads, NULL);
}

/* Natural tile order (0, 1, ..., n-1 in every split). */
int oracle_decode(const oracle_shape* sh, int kind, const void* q, const void* k, const void* v,
                  const uint16_t* k_scale, const uint16_t* v_scale, const int32_t* seq_lens,
                  const oracle_art* art, double tau, const int32_t* forced_used, int no_break,
                  double* o, int32_t* used, int32_t* tiles, double* metrics, int n_threads) {
  return oracle_decode_ordered(sh, kind, q, k, v, k_scale, v_scale, seq_lens, art, tau, forced_used,
                               no_break, NULL, o, used, tiles, metrics, n_threads);
}
