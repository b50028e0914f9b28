"""CPU oracle for the FP8 W8A8 row-wise linear path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library; the only module both sides use is the seeded
input generator package ``workloads``, which holds none of the method's
arithmetic.

The oracle is plain numpy, written for a reader to check against the pages by
eye: FP8 decodes by table, quantization is fp32 IEEE round-to-nearest
arithmetic with a table-search encoder, and the GEMM accumulates in fp64
(exact for these formats and sizes). ``int8`` holds the int8 W8A8 build
(exact integer GEMM), ``w4a16`` the 4-bit build over the exact QAT weights,
``moe`` the mixture-of-experts layer.

Pages cited (by title and section):

* [E2B]  "MI300X 上跑 Gemma 4 E2B：fp8 最快，却离原始权重最远" (geoz.com.cn).
* [SIZES] "Gemma 4 From E2B to 31B on an AMD MI300X: fp8 Overtakes bf16
  From 12B Up" (dev.to).
* [CARD] "Gemma 4 31B-it QAT, FP8 E4M3 W8A8, text only (unofficial)"
  (model card mirror).
* [PR]   "PR #45854 完整报告" (prhub.com.cn, vLLM fp8_per_channel report).

Pin status of every function is listed in the module that defines it; each
function here is pinned by a ``-m "not gpu"`` test in ``tests/`` against
library casts, closed forms or brute force (see ``tests/test_oracle_*.py``).
"""

from .formats import (
    E4M3_MAX,
    E4M3FNUZ_MAX,
    dec_e4m3,
    dec_e4m3fnuz,
    enc_e4m3,
    enc_e4m3fnuz,
)
from .quantize import (
    QuantResult,
    convert_fnuz_to_e4m3,
    fnuz_copy_of_e4m3,
    quant_act,
    quantize_rows,
    quantize_rows_fnuz,
    repack_qat,
    unpack_q4,
    qat_values,
)
from .gemm import rowwise_linear_ref, rowwise_linear_tolerance, check_linear, bf16_ulp
from .formats import bf16_rne_bits
from . import int8, moe, w4a16

__all__ = [
    "E4M3_MAX", "E4M3FNUZ_MAX", "dec_e4m3", "dec_e4m3fnuz", "enc_e4m3", "enc_e4m3fnuz",
    "QuantResult", "convert_fnuz_to_e4m3", "fnuz_copy_of_e4m3", "quant_act",
    "quantize_rows", "quantize_rows_fnuz", "repack_qat", "unpack_q4", "qat_values",
    "rowwise_linear_ref", "rowwise_linear_tolerance", "check_linear", "bf16_ulp", "moe",
    "bf16_rne_bits", "int8", "w4a16",
]
