"""Reader for the hand-derived golden fixtures under tests/golden/.

Each data line is ``name = e1 e2 ...`` where every entry is an arithmetic
expression in rationals and ``ln(.)``.  Expressions are evaluated with a
whitelist (numbers, + - * / and parentheses, ln) so a fixture cannot run code.
"""

import ast
import math
import os

import numpy as np

_ALLOWED = (ast.Expression, ast.BinOp, ast.UnaryOp, ast.Constant, ast.Call,
            ast.Name, ast.Load, ast.Add, ast.Sub, ast.Mult, ast.Div,
            ast.USub, ast.UAdd, ast.Pow)


def _eval(expr: str) -> float:
    tree = ast.parse(expr, mode="eval")
    for node in ast.walk(tree):
        if not isinstance(node, _ALLOWED):
            raise ValueError(f"disallowed token in golden expression: {expr}")
        if isinstance(node, ast.Name) and node.id != "ln":
            raise ValueError(f"unknown name in golden expression: {expr}")
    return float(eval(compile(tree, "<golden>", "eval"), {"__builtins__": {}}, {"ln": math.log}))


def load(path: str) -> dict:
    out = {}
    with open(path) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            name, rhs = line.split("=", 1)
            out[name.strip()] = np.array([_eval(t) for t in rhs.split()], dtype=np.float64)
    return out


def stack(g: dict, prefix: str, n: int) -> np.ndarray:
    return np.stack([g[f"{prefix}{i}"] for i in range(n)])


def golden_path(name: str) -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
