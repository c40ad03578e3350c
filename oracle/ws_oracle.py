"""Plain fp64 CPU oracle of the performer's per-unit denoising step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library: it never loads it, it has its
own bf16 conversion, its own cache model and its own error rules, written from
the pages' description and from the interface specification in ``include/ws.h``.

Sources (the five pages on Wan-Streamer v0.2, cited by page and section):

* [rainbus]  "Wan-Streamer v0.2：更高分辨率，相同延迟" (paper.rainbus.top),
  sections 前置知识 / K/V缓存预分片, 核心方法, 方法步骤详情.
* [remio]    "通义实验室发布 Wan-Streamer v0.2，端到端延迟达 550ms，但由更多 GPU 承担负载"
  (remio.ai), sections 为什么端到端模型对级联式 AI 智能体构成挑战 and
  思考者与执行者的分工掩盖了更高分辨率的成本.
* [gist-en]  "Technical Summary: Wan-Streamer v0.2" (gist.science), section
  Methodology, item 2 (K/V Handling).

What each part follows:

* Cache model (``UnitCache``): the performer keeps a history cache into which
  each incoming thinker K/V slice is written in place [rainbus 前置知识/K/V缓存预分片;
  gist-en Methodology 2]; generated latents are committed back into that
  history after each unit [rainbus 核心方法]; the cache reuses past tokens' K/V
  instead of recomputing them [remio 思考者与执行者…].  The ring of C = U + 1
  unit slots, ``slot(u) = u mod C``, is the reading this build takes of a
  U-unit history held in preallocated memory.
* Attention (``attention_rows``): block-causal attention, block = one 160 ms
  unit: a token sees every token of its own unit and of earlier units, never a
  later one [remio 为什么端到端…].  Within the visible set the operation is the
  plain definition of softmax attention with scale 1/sqrt(D): s_j = q.k_j/sqrt(D),
  p_j = exp(s_j - max s) / sum exp(s - max s), out = sum_j p_j v_j.
* Multi-unit queries (``UnitCache.prefill_attention``): several consecutive
  query units at once, each over its own window, the same block-causal rule
  [remio 为什么端到端…].
* Sessions (``SessionPool``): independent conversations, one UnitCache each,
  batched into one call; every query unit sees its own session only.  How many
  conversations one deployment carries is the question the pages leave open
  [remio 决定 Wan-Streamer 是否重要的三个信号].
* Euler (``euler_step``): one flow-matching update x <- x + dt*v of the
  latent [rainbus 核心方法 (flow-matching latent generation)], evaluated as
  RN_bf16(fl64(x + fl64(dt*v))); dt*v is exact in fp64.

Parity pins (tests/test_oracle_*.py): brute-force full-sequence masked attention
on tiny inputs, R-way splits of rows and heads (bit-identical), softmax row sums,
closed forms (q = 0, constant V, one key, equal keys, two keys with logit gap ln 3),
a torch float64 SDPA witness, exact-rational rounding for the bf16 conversion and
the Euler step, the ring's closed form, per-query-unit brute force for multi-unit
queries, and per-session brute force plus session isolation for batched sessions.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# Status codes of the interface specification (include/ws.h), restated here.
OK = 0
ERR_ARG = -1
ERR_ALIGN = -2
ERR_OOM = -3
ERR_UNIT_ORDER = -4
ERR_EVICTED = -5
ERR_NOT_READY = -6
ERR_UNSUPPORTED = -9
MAX_QUERY_UNITS = 64

SEG_COND = 0
SEG_LATENT = 1


# ---------------------------------------------------------------- bf16 ----

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly (bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):                  # signalling NaN patterns
        return b.view(np.float32).astype(np.float64)


_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def f64_to_bf16(x) -> np.ndarray:
    """Round float64 to bf16 bit patterns, round-to-nearest-even (IEEE 754 default).

    bf16 keeps 8 significant bits and fp32's exponent range.  A value in
    [2^(e-1), 2^e) has quantum 2^(e-8); below 2^-126 the quantum is the
    subnormal step 2^-133.  x / quantum is rounded half-to-even by ``np.rint``
    (scaling by a power of two is exact), and magnitudes past the largest
    finite bf16 after rounding become infinities.  Every NaN maps to the
    positive quiet NaN 0x7FC0 (the sign of a NaN is not significant and
    differs between processors).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    finite = np.isfinite(x)
    _, e = np.frexp(np.where(finite, x, 0.0))              # x = m * 2^e, m in [0.5, 1)
    qexp = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(np.where(finite, x, 0.0), -qexp)), qexp)
    over = np.abs(y) > _BF16_MAX
    y = np.where(over, np.copysign(np.inf, y), y)
    out[...] = (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    out[np.isnan(x)] = 0x7FC0          # every NaN becomes the positive quiet NaN
    inf = np.isinf(x)
    out[inf] = np.where(x[inf] > 0, 0x7F80, 0xFF80)
    return out


# ---------------------------------------------------------------- Euler ---

def euler_step(x_bits, v_bits, dt: float) -> np.ndarray:
    """One flow-matching Euler update of a bf16 latent: RN_bf16(x + dt*v).

    ``dt`` is an fp32 value (the interface passes a C float); the product of an
    fp32 and a bf16 fits in fp64 exactly, the sum is rounded once to fp64 and
    once to bf16.
    """
    dt64 = np.float64(np.float32(dt))
    return f64_to_bf16(bf16_to_f64(x_bits) + dt64 * bf16_to_f64(v_bits))


# ------------------------------------------------------------ attention ---

def attention_rows(q, k, v, rows=None, heads=None, return_probs=False):
    """Softmax attention of every (head, query row) over all given keys.

    q: [Nq, H, D], k and v: [Nk, H, D] (float64 or anything convertible).
    Each (head, row) is computed on its own, so the result of a row never
    depends on which other rows or heads are asked for.
    Returns out [len(rows), len(heads), D] (and probs [len(rows), len(heads), Nk]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nh, d = q.shape
    rows = range(nq) if rows is None else rows
    heads = range(nh) if heads is None else heads
    rows, heads = list(rows), list(heads)
    scale = 1.0 / math.sqrt(d)
    out = np.empty((len(rows), len(heads), d))
    probs = np.empty((len(rows), len(heads), k.shape[0])) if return_probs else None
    for hi, h in enumerate(heads):
        kh = np.ascontiguousarray(k[:, h, :])
        vh = np.ascontiguousarray(v[:, h, :])
        for ri, i in enumerate(rows):
            s = (kh @ q[i, h, :]) * scale
            e = np.exp(s - s.max())
            p = e / e.sum()
            out[ri, hi, :] = p @ vh
            if return_probs:
                probs[ri, hi, :] = p
    return (out, probs) if return_probs else out


# ----------------------------------------------------------- cache model --

@dataclass
class Config:
    n_layers: int
    n_heads: int
    head_dim: int
    n_video: int
    n_audio: int
    n_cond: int
    history_units: int

    @property
    def n_query(self) -> int:          # latent tokens generated per unit
        return self.n_video + self.n_audio

    @property
    def tokens_per_unit(self) -> int:  # T = cond + latent
        return self.n_cond + self.n_query

    @property
    def slots(self) -> int:            # C = U + 1
        return self.history_units + 1


@dataclass
class _Unit:
    cond_k: np.ndarray                         # [L, Nc, H, D] bf16 bits
    cond_v: np.ndarray
    lat_k: dict = field(default_factory=dict)  # layer -> [Nq, H, D] bf16 bits
    lat_v: dict = field(default_factory=dict)


class UnitCache:
    """Logical model of the performer's K/V history.

    Units arrive in non-decreasing order.  Appending the conditioning slice of a
    new unit u claims slot ``u mod C`` and so evicts whatever unit held it.  A
    unit's latent K/V of a layer exists once it has been written, either by the
    attention call of that layer (the current, still-noisy latent) or by the
    all-layer commit.  Attention for the newest unit u sees, for every resident
    unit u' with u - U <= u' <= u, the conditioning tokens of u' and the latent
    tokens of u' for that layer if written.
    """

    def __init__(self, cfg: Config):
        self.cfg = cfg
        self.units: dict[int, _Unit] = {}
        self.slot_unit = [-1] * cfg.slots
        self.newest = -1

    # -- bookkeeping ------------------------------------------------------
    def slot(self, unit: int) -> int:
        return unit % self.cfg.slots

    def _resident(self, unit: int) -> int:
        if unit < 0:
            return ERR_ARG
        holder = self.slot_unit[self.slot(unit)]
        if holder == unit:
            return OK
        return ERR_EVICTED if holder > unit else ERR_NOT_READY

    def slot_table(self) -> list[int]:
        return list(self.slot_unit)

    # -- writes -----------------------------------------------------------
    def append(self, unit: int, seg: int, k_bits, v_bits) -> int:
        c = self.cfg
        if seg == SEG_COND:
            shape = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
            if unit < 0 or np.shape(k_bits) != shape or np.shape(v_bits) != shape:
                return ERR_ARG
            if unit < self.newest:
                return ERR_UNIT_ORDER
            if unit > self.newest:
                old = self.slot_unit[self.slot(unit)]
                self.units.pop(old, None)
                self.slot_unit[self.slot(unit)] = unit
                self.units[unit] = _Unit(np.array(k_bits, dtype=np.uint16), np.array(v_bits, dtype=np.uint16))
                self.newest = unit
            else:
                self.units[unit].cond_k = np.array(k_bits, dtype=np.uint16)
                self.units[unit].cond_v = np.array(v_bits, dtype=np.uint16)
            return OK
        if seg == SEG_LATENT:
            shape = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
            if unit < 0 or np.shape(k_bits) != shape or np.shape(v_bits) != shape:
                return ERR_ARG
            st = self._resident(unit)
            if st != OK:
                return st
            u = self.units[unit]
            for l in range(c.n_layers):
                u.lat_k[l] = np.array(k_bits[l], dtype=np.uint16)
                u.lat_v[l] = np.array(v_bits[l], dtype=np.uint16)
            return OK
        return ERR_ARG

    def read(self, layer: int, unit: int, seg: int):
        """(status, k, v) of one segment of one unit and layer, as bf16 bits."""
        c = self.cfg
        if not (0 <= layer < c.n_layers) or seg not in (SEG_COND, SEG_LATENT):
            return ERR_ARG, None, None
        st = self._resident(unit)
        if st != OK:
            return st, None, None
        u = self.units[unit]
        if seg == SEG_COND:
            return OK, u.cond_k[layer], u.cond_v[layer]
        if layer not in u.lat_k:
            return ERR_NOT_READY, None, None
        return OK, u.lat_k[layer], u.lat_v[layer]

    # -- the hot path -----------------------------------------------------
    def visible_units(self, unit: int) -> list[int]:
        lo = unit - self.cfg.history_units
        return sorted(u for u in self.units if lo <= u <= unit)

    def visible_kv(self, layer: int, unit: int):
        """Keys and values (float64, [Nk, H, D]) the query unit sees at ``layer``,
        plus the unit index of every key."""
        ks, vs, owner = [], [], []
        for u in self.visible_units(unit):
            rec = self.units[u]
            ks.append(bf16_to_f64(rec.cond_k[layer]))
            vs.append(bf16_to_f64(rec.cond_v[layer]))
            owner += [u] * rec.cond_k.shape[1]
            if layer in rec.lat_k:
                ks.append(bf16_to_f64(rec.lat_k[layer]))
                vs.append(bf16_to_f64(rec.lat_v[layer]))
                owner += [u] * rec.lat_k[layer].shape[0]
        return np.concatenate(ks), np.concatenate(vs), np.array(owner)

    def unit_attention(self, layer: int, unit: int, q_bits, k_new_bits, v_new_bits,
                       rows=None, heads=None):
        """Write the current unit's latent K/V of ``layer`` and attend.

        Returns (status, out) with out [rows, heads, D] float64.
        """
        c = self.cfg
        shape = (c.n_query, c.n_heads, c.head_dim)
        if not (0 <= layer < c.n_layers) or any(np.shape(a) != shape for a in (q_bits, k_new_bits, v_new_bits)):
            return ERR_ARG, None
        if unit < 0:
            return ERR_ARG, None
        if unit > self.newest:
            return ERR_NOT_READY, None
        if unit < self.newest:
            return ERR_UNIT_ORDER, None
        rec = self.units[unit]
        rec.lat_k[layer] = np.array(k_new_bits, dtype=np.uint16)
        rec.lat_v[layer] = np.array(v_new_bits, dtype=np.uint16)
        k, v, _ = self.visible_kv(layer, unit)
        return OK, attention_rows(bf16_to_f64(q_bits), k, v, rows=rows, heads=heads)


    def prefill_attention(self, layer: int, unit_first: int, n_units: int, q_bits, k_new_bits, v_new_bits,
                          rows=None, heads=None):
        """Several consecutive query units at once (a prompt prefill): write each
        unit's latent K/V of ``layer``, then every query unit attends over its own
        window -- block-causal across units.  q, k_new, v_new: [n, Nq, H, D].

        Every query unit must be resident, the last one the newest, and no unit
        inside a query window may have been overwritten.
        Returns (status, out [n, rows, heads, D] float64)."""
        c = self.cfg
        shape = (n_units, c.n_query, c.n_heads, c.head_dim)
        if not (0 <= layer < c.n_layers) or unit_first < 0 or n_units < 1:
            return ERR_ARG, None
        if n_units > MAX_QUERY_UNITS:
            return ERR_UNSUPPORTED, None
        if any(np.shape(a) != shape for a in (q_bits, k_new_bits, v_new_bits)):
            return ERR_ARG, None
        u_last = unit_first + n_units - 1
        if u_last > self.newest:
            return ERR_NOT_READY, None
        if u_last < self.newest:
            return ERR_UNIT_ORDER, None
        for u in range(unit_first, u_last + 1):
            st = self._resident(u)
            if st != OK:
                return st, None
        for u in range(max(0, unit_first - self.cfg.history_units), unit_first):
            if self.slot_unit[self.slot(u)] > u:
                return ERR_EVICTED, None
        for j in range(n_units):
            rec = self.units[unit_first + j]
            rec.lat_k[layer] = np.array(k_new_bits[j], dtype=np.uint16)
            rec.lat_v[layer] = np.array(v_new_bits[j], dtype=np.uint16)
        outs = []
        for j in range(n_units):
            k, v, _ = self.visible_kv(layer, unit_first + j)
            outs.append(attention_rows(bf16_to_f64(q_bits[j]), k, v, rows=rows, heads=heads))
        return OK, np.stack(outs)


class SessionPool:
    """Several independent conversations served together (session economics:
    remio.ai, section 决定 Wan-Streamer 是否重要的三个信号).  Each session is
    its own UnitCache; one batched attention call takes query units of several
    sessions, and each sees its own session's window only.

    Query unit j of a call is (sessions[j], units[j]).  The units of one session
    form a single stretch of consecutive units in the list, ending at that
    session's newest unit; each stretch follows that session's prefill rules.
    The list is checked stretch by stretch in order, and the first failing rule
    gives the status.
    """

    def __init__(self, cfg: Config, n_sessions: int):
        self.cfg = cfg
        self.sessions = [UnitCache(cfg) for _ in range(n_sessions)]

    def reset(self, session: int) -> int:
        """The session's conversation ends; its ring starts empty."""
        if not 0 <= session < len(self.sessions):
            return ERR_ARG
        self.sessions[session] = UnitCache(self.cfg)
        return OK

    def session_attention(self, layer: int, sessions, units, q_bits, k_new_bits, v_new_bits,
                          rows=None, heads=None):
        """Returns (status, out [n, rows, heads, D] float64)."""
        c = self.cfg
        n = len(sessions)
        if not (0 <= layer < c.n_layers) or n < 1 or len(units) != n:
            return ERR_ARG, None
        if n > MAX_QUERY_UNITS:
            return ERR_UNSUPPORTED, None
        shape = (n, c.n_query, c.n_heads, c.head_dim)
        if any(np.shape(a) != shape for a in (q_bits, k_new_bits, v_new_bits)):
            return ERR_ARG, None
        if any(not 0 <= s < len(self.sessions) for s in sessions) or any(u < 0 for u in units):
            return ERR_ARG, None
        stretches, seen, j = [], set(), 0
        while j < n:
            s = sessions[j]
            if s in seen:
                return ERR_ARG, None
            seen.add(s)
            k = j
            while k + 1 < n and sessions[k + 1] == s:
                if units[k + 1] != units[k] + 1:
                    return ERR_ARG, None
                k += 1
            cache = self.sessions[s]
            u_first, u_last = units[j], units[k]
            if u_last > cache.newest:
                return ERR_NOT_READY, None
            if u_last < cache.newest:
                return ERR_UNIT_ORDER, None
            for u in range(u_first, u_last + 1):
                st = cache._resident(u)
                if st != OK:
                    return st, None
            for u in range(max(0, u_first - c.history_units), u_first):
                if cache.slot_unit[cache.slot(u)] > u:
                    return ERR_EVICTED, None
            stretches.append((s, j, k))
            j = k + 1
        out = [None] * n
        for s, j, k in stretches:
            st, o = self.sessions[s].prefill_attention(layer, units[j], k - j + 1, q_bits[j:k + 1],
                                                       k_new_bits[j:k + 1], v_new_bits[j:k + 1],
                                                       rows=rows, heads=heads)
            assert st == OK
            for i in range(k - j + 1):
                out[j + i] = o[i]
        return OK, np.stack(out)


def attention_flops(n_query: int, n_keys: int, n_heads: int, head_dim: int) -> float:
    """Algorithmic FLOPs of one attention call: QK^T and PV, 2 FLOPs per multiply-add."""
    return 4.0 * n_query * n_keys * n_heads * head_dim
