"""CPU reference (the oracle) of the decode step.  TEST INFRASTRUCTURE ONLY:
only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import it.  It shares no code with the CUDA path."""
from .oracle import (OracleModel, OracleState, build, lib, load_variant, compile_variant,
                     source_text, attend, attend_split, gemv, rmsnorm, rope, softmax, silu,
                     argmax, bf16_round, kv_cache_bytes, num_threads, quantize_fp8_rows,
                     quantize_fp8_model)

__all__ = ["OracleModel", "OracleState", "build", "lib", "load_variant", "compile_variant",
           "source_text", "attend", "attend_split", "gemv", "rmsnorm", "rope", "softmax", "silu",
           "argmax", "bf16_round", "kv_cache_bytes", "num_threads", "quantize_fp8_rows",
           "quantize_fp8_model"]
