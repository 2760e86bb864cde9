"""Test-infrastructure oracle: an fp64 CPU restatement of the packed DiT
block.  Only tests, the smoke check and the bench's CPU baseline import it."""
