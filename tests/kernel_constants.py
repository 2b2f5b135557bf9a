"""Barrier arrive counts and ring depths of the tcgen05 kernels, read out of
their CUDA sources.

The CPU protocol models (tests/test_*_protocol.py) take their ring depths and
barrier counts from here instead of restating them, so a change to a kernel's
`mbar_init` counts or stage depth changes the model with it (and a count the
model cannot map to its roles fails the model's constants test).  Pure text
parsing: nothing here loads or runs the library.
"""
from __future__ import annotations

import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_io_aware_55_b200", "csrc")

# Values of the symbolic names the counts and depths are written with.
_SYMBOLS = {"kNQT": 2}


def _source(name: str) -> str:
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _eval(expr: str, extra=None) -> int:
    env = dict(_SYMBOLS)
    env.update(extra or {})
    expr = expr.strip()
    if not re.fullmatch(r"[\w\s+\-*/()]+", expr):
        raise ValueError(f"unexpected count expression {expr!r}")
    return int(eval(expr, {"__builtins__": {}}, env))  # noqa: S307 -- arithmetic on known names only


def _literal_constants(src: str) -> dict[str, int]:
    """`constexpr int NAME = <integer literal>;` definitions of a source file."""
    return {m.group(1): int(m.group(2)) for m in re.finditer(r"constexpr int (\w+)\s*=\s*(\d+)\s*;", src)}


def barrier_counts(name: str) -> dict[str, int]:
    """{barrier: arrive count} from every `mbar_init(&<obj>-><barrier>[...]..., count)`
    in the source file (array barriers share one count; the last init wins)."""
    src = _source(name)
    env = {}
    for inc in re.findall(r'#include "([\w.]+)"', src):   # constants of the file's own headers
        if os.path.exists(os.path.join(CSRC, inc)):
            env.update(_literal_constants(_source(inc)))
    env.update(_literal_constants(src))
    out = {}
    for m in re.finditer(r"mbar_init\(&\w+->(\w+)(?:\[[^\]]*\])*,\s*([^;]+?)\);", src):
        out[m.group(1)] = _eval(m.group(2), env)
    if not out:
        raise ValueError(f"no mbar_init found in {name}")
    return out


def ring_depth(name: str, symbol: str, d: int | None = None) -> int:
    """Value of `constexpr int <symbol> = <expr>;` in the source file; `d` (head
    dimension) resolves expressions that depend on D or the tile size."""
    m = re.search(r"constexpr int " + re.escape(symbol) + r"\s*=\s*([^;]+);", _source(name))
    if not m:
        raise ValueError(f"{symbol} not found in {name}")
    expr = m.group(1)
    extra = {}
    if d is not None:
        extra["D"] = d
        extra["kTileBytes"] = 128 * d * 2
    t = re.fullmatch(r"\((.+?)\s*(>=|==)\s*(\w+)\)\s*\?\s*(\w+)\s*:\s*(\w+)", expr.strip())
    if t:   # a conditional: (a >= b) ? x : y  /  (a == b) ? x : y
        a, op, b, x, y = t.groups()
        av, bv = _eval(a, extra), _eval(b, extra)
        return _eval(x if (av >= bv if op == ">=" else av == bv) else y, extra)
    return _eval(expr, extra)


def per_agent(count: int, arrivals_per_agent: int, what: str) -> int:
    """Model count for a barrier whose agents each stand for
    `arrivals_per_agent` arriving warps (or threads) of the kernel."""
    if count % arrivals_per_agent:
        raise ValueError(f"{what}: kernel count {count} is not a multiple of {arrivals_per_agent}")
    return count // arrivals_per_agent
