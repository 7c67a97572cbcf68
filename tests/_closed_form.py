"""Evaluate the golden fixtures' closed-form expressions with Python's decimal module.

Independent of numpy and of the oracle: 40-digit decimal arithmetic with
exp, ln and sqrt taken from the decimal module itself.
"""
import ast
import json
import os
from decimal import Decimal, getcontext

getcontext().prec = 40

_FUNCS = {
    "exp": lambda v: v.exp(),
    "ln": lambda v: v.ln(),
    "sqrt": lambda v: v.sqrt(),
}


def _ev(node):
    if isinstance(node, ast.Expression):
        return _ev(node.body)
    if isinstance(node, ast.Constant):
        return Decimal(str(node.value))
    if isinstance(node, ast.UnaryOp) and isinstance(node.op, ast.USub):
        return -_ev(node.operand)
    if isinstance(node, ast.BinOp):
        a, b = _ev(node.left), _ev(node.right)
        if isinstance(node.op, ast.Add):
            return a + b
        if isinstance(node.op, ast.Sub):
            return a - b
        if isinstance(node.op, ast.Mult):
            return a * b
        if isinstance(node.op, ast.Div):
            return a / b
        if isinstance(node.op, ast.Pow):
            return a ** b
    if isinstance(node, ast.Call) and isinstance(node.func, ast.Name) and node.func.id in _FUNCS:
        return _FUNCS[node.func.id](_ev(node.args[0]))
    raise ValueError(f"unsupported expression node {ast.dump(node)}")


def ev(expr) -> Decimal:
    """Exact-ish (40 digits) value of an expression string such as 'sqrt(ln(2))'."""
    return _ev(ast.parse(str(expr), mode="eval"))


def evf(expr) -> float:
    return float(ev(expr))


def load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)
