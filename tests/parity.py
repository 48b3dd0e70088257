"""The row comparison lives with the oracle (oracle/parity.py), so that the
smoke check and the benchmark's CPU leg can report the same figures."""
from oracle.parity import RECORDS, check_rows  # noqa: F401
