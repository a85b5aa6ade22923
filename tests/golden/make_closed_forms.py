"""Write the closed-form fixtures in this folder.

Every stored value follows from a mathematical definition, evaluated here in
exact or 40-digit decimal arithmetic; nothing comes from the oracle or the
CUDA path.  Run:  python tests/golden/make_closed_forms.py
"""
import json
import os
from decimal import Decimal, getcontext

getcontext().prec = 40
HERE = os.path.dirname(os.path.abspath(__file__))


def write(name, obj):
    with open(os.path.join(HERE, name), "w") as f:
        json.dump(obj, f, indent=1)
        f.write("\n")


def bf16_cases():
    # Exact binary values on and around rounding boundaries of bfloat16.
    c = [
        ("1 + 2^-8 (tie between 1 and 1 + 2^-7): ties to even -> 1", 1 + 2**-8, 0x3F80),
        ("1 + 3*2^-8 (tie): ties to even -> 1 + 2^-6", 1 + 3 * 2**-8, 0x3F82),
        ("just above the tie 1 + 2^-8 rounds up", 1 + 2**-8 + 2**-40, 0x3F81),
        ("-(1 + 2^-8) ties to even, sign kept", -(1 + 2**-8), 0xBF80),
        ("largest finite bf16 (2 - 2^-7) * 2^127", (2 - 2**-7) * 2**127, 0x7F7F),
        ("(2 - 2^-8) * 2^127 is the tie to 2^128: rounds to even -> inf", (2 - 2**-8) * 2**127, 0x7F80),
        ("just below that tie stays finite", (2 - 2**-8) * 2**127 - 2**100, 0x7F7F),
        ("smallest normal 2^-126", 2**-126, 0x0080),
        ("smallest subnormal 2^-133", 2**-133, 0x0001),
        ("2^-134 is the tie between 0 and 2^-133: ties to even -> +0", 2**-134, 0x0000),
        ("3 * 2^-134 is the tie between 2^-133 and 2^-132: ties to even -> 2^-132", 3 * 2**-134, 0x0002),
        ("pi = 3.14159... rounds to 3.140625 (0x4049)", 3.141592653589793, 0x4049),
        ("0.1 rounds to 0.10009765625 (0x3DCD)", 0.1, 0x3DCD),
        ("-0.0 keeps its sign", -0.0, 0x8000),
    ]
    return {"source": "bfloat16 = the upper 16 bits of IEEE 754 binary32 (1 sign, 8 exponent, 7 fraction "
                      "bits); round to nearest, ties to even (IEEE 754-2019, clause 4.3.1); each case is "
                      "derived by hand from that definition",
            "cases": [{"what": w, "x": float.hex(float(x)), "bits": b} for w, x, b in c]}


def rope_cases():
    # theta^(-2j/d) with theta = 10^4 is 10^(-8j/d): a power of ten when 8j/d is an integer.
    c = []
    for d, j, what in [(128, 0, "first pair rotates by the position itself"),
                       (128, 16, "10000^(-32/128) = 10^-1"), (128, 32, "10000^(-64/128) = 10^-2"),
                       (128, 48, "10000^(-96/128) = 10^-3"), (64, 8, "10000^(-16/64) = 10^-1"),
                       (64, 16, "10000^(-32/64) = 10^-2"),
                       (44, 11, "3D t-section of 44 elements: 10000^(-22/44) = 10^-2"),
                       (42, 0, "first pair of a 42-wide section")]:
        exp10 = Decimal(-8 * j) / Decimal(d)
        assert exp10 == exp10.to_integral_value()
        c.append({"d": d, "j": j, "freq": float(Decimal(10) ** exp10), "what": what})
    return {"source": "rotary position embedding frequency theta^(-2j/d) (RoFormer, Su et al. 2021, "
                      "section 3.2.2) with theta = 10000; closed-form points where 8j/d is an integer",
            "theta": 10000.0, "cases": c}


def silu_cases():
    c = []
    for a in ["0", "1", "-1", "2", "-2", "0.5", "-0.5", "4"]:
        A = Decimal(a)
        s = A / (1 + (-A).exp())
        c.append({"a": float(A), "silu": float(s), "silu_40": str(s)})
    return {"source": "SiLU / swish: silu(a) = a / (1 + exp(-a)) (Elfwing et al. 2018); evaluated with "
                      "40-digit decimal arithmetic", "cases": c}


if __name__ == "__main__":
    write("bf16_rounding.json", bf16_cases())
    write("rope_frequencies.json", rope_cases())
    write("silu_closed_forms.json", silu_cases())
